"""Benchmark of the QLoRA NF4 + LoRA quantized linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass over every part of the hot path on synthetic inputs
already resident in HBM:

  1. quantize the 7B-MLP-shaped weight W [11008 x 4096] to NF4 + double quant
  2. forward  y = x W_hat^T + s (x A^T) B^T      (x: 4096 tokens, r = 64, alpha = 16)
  3. backward dX, dA, dB                          (dY: 4096 x 11008)
  4. decode forward (GEMV) on a resident 4096 x 4096 NF4 weight, 1 token

The headline ``value`` is the algorithmic forward + backward FLOPs of steps 2-3
divided by the device time of the whole step (quantize and decode included),
in TFLOP/s, summed over ranks (weak scaling: every rank runs its own 4096
tokens; the LoRA gradients are all-reduced over NCCL, the data-parallel
exchange). L2 is flushed (256 MiB write) before every timed step, outside the
timed events. Extra keys report each part, the decode GEMV in steady state (a
CUDA graph of back-to-back calls over 32 rotating weight copies, > 2x L2), the
end-to-end number through host buffers, the oracle timed on the host cores,
and the roofline of the dominant call.

``--impl reference`` times the CPU oracle (the plain fp64 statement of the
method) on a bounded sample of the same workload.
"""

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "NF4+LoRA linear fwd/bwd TFLOP/s and dequant-GEMV GB/s (% of B200 roofline)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of one 7B-MLP forward call (its three launches),
# from one ncu capture, and a digest of the sources that build those kernels
# at capture time. If any of them has changed since, the figure no longer
# describes the kernel that runs and the roofline's traffic is reported null.
FWD_TRAFFIC = {"bytes": 161873664, "sources_sha256": "1b443ce2020f123c58fa76856b5cadb984f9884b3be7dbda88bca0a46ec5d036",
               "profile": "profiles/qlora_linear_fwd_bwd_7b_mlp_dram.md"}
FWD_SOURCES = ["api.cu", "tc_pair.cu", "tc_gemm.cu", "kernels.h", "ptx.cuh", "nf4_dev.cuh", "tc_common.cuh", "pair_sched.h"]


def fwd_sources_digest():
    import hashlib
    h = hashlib.sha256()
    for f in FWD_SOURCES:
        with open(os.path.join(ROOT, "bit_nf4_quantized_06_b200", "csrc", f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()


def fwd_traffic():
    if FWD_TRAFFIC["bytes"] is None or FWD_TRAFFIC["sources_sha256"] != fwd_sources_digest():
        return None
    return FWD_TRAFFIC["bytes"]


# ----------------------------------------------------------------------------- workload arithmetic
def fwd_flops(m, n, k, r):
    """Algorithmic forward FLOPs: x W^T, x A^T, u' B^T."""
    return 2.0 * m * n * k + 2.0 * m * k * r + 2.0 * m * r * n


def bwd_flops(m, n, k, r):
    """dX = dY W + v' A with v' = dY B, dA = v'^T x, dB = dY^T u'."""
    return 2.0 * m * n * k + 2.0 * m * n * r + 2.0 * m * r * k + 2.0 * m * r * k + 2.0 * m * n * r


def gemv_bytes(n, k, r, m=1):
    """Algorithmic bytes of one decode call: packed W, scale codes, s_max, A, B, x, y."""
    nb = n * k // 64
    return n * k // 2 + nb + 4 * math.ceil(nb / 256) + 2 * r * (k + n) + 2 * m * (k + n)


def quant_bytes(n, k):
    """Algorithmic bytes of the quantizer: read bf16 W, write codes, scale codes, s_max."""
    nb = n * k // 64
    return 2 * n * k + n * k // 2 + nb + 4 * math.ceil(nb / 256)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"]))}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value, world):
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_grads(tensors, world):
    """Data-parallel exchange of the LoRA gradients: sum over ranks, then mean."""
    if world <= 1:
        return
    import torch.distributed as dist
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        t.div_(world)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, busy_only=True):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5], parts[6], parts[7],
                             parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return out
        loaded = [r for r in rows if r[2] > 250.0] if busy_only else rows
        use = loaded or rows
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in use:
            for nm, v in zip(names, r[3:]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        out.update({"sm_mhz": float(np.median([r[0] for r in use])), "sm_max_mhz": max(r[1] for r in use),
                    "reasons": sorted(reasons), "samples": len(use)})
        return out


# ----------------------------------------------------------------------------- our arm
class Workload:
    def __init__(self, q, device, rank):
        p, d = synth.MLP7B, synth.DECODE
        self.q, self.p, self.d = q, p, d
        seed = 1000 * rank
        t = synth.make(p, seed=seed)
        self.host = {k: v.pin_memory() for k, v in t.items()}
        self.w = t["w"].to(device)
        self.x = t["x"].to(device)
        self.a = t["a"].to(device)
        self.b = t["b"].to(device)
        self.dy = t["dy"].to(device)
        self.qw = q.NF4Weight(p.n, p.k, device=device)
        self.y = torch.empty((p.m, p.n), dtype=torch.bfloat16, device=device)
        self.u = torch.empty((p.m, p.r), dtype=torch.bfloat16, device=device)
        self.dx = torch.empty((p.m, p.k), dtype=torch.bfloat16, device=device)
        self.da = torch.empty((p.r, p.k), dtype=torch.float32, device=device)
        self.db = torch.empty((p.n, p.r), dtype=torch.float32, device=device)
        self.ws = torch.empty(q.qlora_workspace_bytes(p.m, p.n, p.k, p.r) + 256, dtype=torch.uint8, device=device)
        # decode: resident packed weight (quantized once, like a loaded model)
        td = synth.make(d, seed=seed + 7)
        self.dec_host_x = td["x"].pin_memory()
        self.dw = q.qlora_quantize_nf4(td["w"].to(device))
        self.dx_in = td["x"].to(device)
        self.da_ = td["a"].to(device)
        self.db_ = td["b"].to(device)
        self.dy_out = torch.empty((d.m, d.n), dtype=torch.bfloat16, device=device)
        self.dws = torch.empty(q.qlora_workspace_bytes(d.m, d.n, d.k, d.r) + 256, dtype=torch.uint8, device=device)
        self.flops = fwd_flops(p.m, p.n, p.k, p.r) + bwd_flops(p.m, p.n, p.k, p.r)

    def step(self, world, ev=None):
        q, p, d = self.q, self.p, self.d
        if ev is not None:
            ev[0].record()
        q.qlora_quantize_nf4(self.w, out=self.qw)
        if ev is not None:
            ev[1].record()
        q.qlora_linear_fwd(self.qw, self.x, self.a, self.b, p.alpha, y=self.y, u=self.u, ws=self.ws)
        if ev is not None:
            ev[2].record()
        q.qlora_linear_bwd(self.qw, self.x, self.u, self.dy, self.a, self.b, p.alpha, dx=self.dx, da=self.da,
                           db=self.db, ws=self.ws)
        allreduce_grads([self.da, self.db], world)
        if ev is not None:
            ev[3].record()
        q.qlora_linear_fwd(self.dw, self.dx_in, self.da_, self.db_, d.alpha, y=self.dy_out, ws=self.dws,
                           want_u=False)
        if ev is not None:
            ev[4].record()


def flush_l2(buf):
    buf.add_(1)


def e2e_pipelined(wl, steps, world, h2d, d2h):
    """Per-step time of `steps` steps through host buffers: each step's inputs
    are copied H2D from pinned memory on a copy stream (into the set of device
    buffers the step before did not use, once that step is done with it) while
    the previous step computes, and each step's results are read back D2H into
    pinned memory. One event pair around all steps (the first copy included),
    max over ranks."""
    dev = wl.x.device
    names = ("x", "dy", "w", "dx_in")
    sets = [{k: getattr(wl, k) for k in names}, {k: torch.empty_like(getattr(wl, k)) for k in names}]
    host = {"x": wl.host["x"], "dy": wl.host["dy"], "w": wl.host["w"], "dx_in": wl.dec_host_x}
    out_da = torch.empty(wl.da.shape, dtype=torch.float32).pin_memory()
    out_db = torch.empty(wl.db.shape, dtype=torch.float32).pin_memory()
    out_y = torch.empty(wl.dy_out.shape, dtype=torch.bfloat16).pin_memory()
    main = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(device=dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def fill(j):
        with torch.cuda.stream(copy):
            for k in names:
                sets[j][k].copy_(host[k], non_blocking=True)
            copied[j].record(copy)

    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e_s.record(main)
    copy.wait_stream(main)
    fill(0)
    for i in range(steps):
        cur, nxt = i % 2, 1 - i % 2
        if i + 1 < steps:
            if i >= 1:
                copy.wait_event(used[nxt])      # step i - 1 is done with that set
            fill(nxt)
        main.wait_event(copied[cur])
        for k in names:
            setattr(wl, k, sets[cur][k])
        wl.step(world)
        used[cur].record(main)
        out_da.copy_(wl.da, non_blocking=True)
        out_db.copy_(wl.db, non_blocking=True)
        out_y.copy_(wl.dy_out, non_blocking=True)
    e_e.record(main)
    torch.cuda.synchronize()
    for k in names:
        setattr(wl, k, sets[0][k])
    return max_over_ranks(e_s.elapsed_time(e_e) / steps, world)


DECODE65 = synth.Problem("decode-gemv-22016x8192-m1-r64", 22016, 8192, 1, 64, 16.0, backward=False)


def gemv_steady_state(q, device, calls=200, copies=32, d=synth.DECODE):
    """Decode GEMV per call in steady state: a CUDA graph of `calls` back-to-back
    forwards cycling over `copies` packed weights (> 2x L2)."""
    t = synth.make(d, seed=77)
    x, a, b = t["x"].to(device), t["a"].to(device), t["b"].to(device)
    w0 = q.qlora_quantize_nf4(t["w"].to(device))
    ws = [q.NF4Weight(d.n, d.k, device=device) for _ in range(copies)]
    for w in ws:
        w.codes.copy_(w0.codes)
        w.scale_codes.copy_(w0.scale_codes)
        w.absmax.copy_(w0.absmax)
    y = torch.empty((d.m, d.n), dtype=torch.bfloat16, device=device)
    work = torch.empty(q.qlora_workspace_bytes(d.m, d.n, d.k, d.r) + 256, dtype=torch.uint8, device=device)
    s = torch.cuda.Stream(device=device)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(3):
            q.qlora_linear_fwd(ws[i % copies], x, a, b, d.alpha, y=y, ws=work, want_u=False, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(calls):
            q.qlora_linear_fwd(ws[i % copies], x, a, b, d.alpha, y=y, ws=work, want_u=False, stream=s)
    launches0 = q.qlora_launch_count()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 5
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * calls)
    # single-call latency, cold weight copy, plain launches
    lat = []
    for i in range(10):
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2.record()
        q.qlora_linear_fwd(ws[(i * 7) % copies], x, a, b, d.alpha, y=y, ws=work, want_u=False)
        e3.record()
        torch.cuda.synchronize()
        lat.append(e2.elapsed_time(e3))
    del g
    return ms, float(np.median(lat)), launches0


def merge_bytes(n, k, r):
    """Algorithmic bytes of one merge: codes, scale codes, group constants, A, B read; bf16 W written."""
    nb = n * k // 64
    return n * k // 2 + nb + 4 * ((nb + 255) // 256) + 2 * r * (k + n) + 2 * n * k


def merge_timing(q, wl, l2, reps=10):
    """LoRA merge for export on the resident 7B-MLP packed weight (L2 flushed before each call)."""
    p = wl.p
    out = torch.empty((p.n, p.k), dtype=torch.bfloat16, device=wl.x.device)
    q.qlora_merge_lora(wl.qw, wl.a, wl.b, p.alpha, out=out)
    times = []
    for _ in range(reps):
        flush_l2(l2)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        q.qlora_merge_lora(wl.qw, wl.a, wl.b, p.alpha, out=out)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = float(np.median(times))
    return ms, merge_bytes(p.n, p.k, p.r)


def paged_optimizer(q, wl, l2, reps=10):
    """AdamW for one adapter pair (A: r x K, B: N x r, 966,656 parameters at
    the 7B-MLP shape) with m, v paged out to pinned host memory, two ways:
    the GPU kernel reading the host states over the link, and the pages' own
    scheme (gradient copied to the host, update on the CPU as a host function
    of a side stream, bf16 adapter copied back). Each is timed alone and as
    the update of "the layer before" running on a second stream beside a
    step's backward (as in a stack, where layer L's update overlaps layer
    L-1's backward); the loss is the step time it adds."""
    p, dev = wl.p, wl.x.device
    n = p.r * p.k + p.n * p.r
    hp = dict(lr=1e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0)
    master = torch.randn(n, device=dev) * 0.01
    param = torch.empty(n, dtype=torch.bfloat16, device=dev)
    grad = torch.randn(n, device=dev) * 1e-3
    m_h, v_h = torch.zeros(n).pin_memory(), torch.zeros(n).pin_memory()
    m_d, v_d = torch.zeros(n, device=dev), torch.zeros(n, device=dev)
    master_h = (torch.randn(n) * 0.01).pin_memory()
    grad_h = torch.empty(n).pin_memory()
    param_h = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    side = torch.cuda.Stream(device=dev)

    def gpu_host_states(i, stream=None):
        q.qlora_adamw_step(master, grad, m_h, v_h, i + 1, param=param, stream=stream, **hp)

    def gpu_device_states(i, stream=None):
        q.qlora_adamw_step(master, grad, m_d, v_d, i + 1, param=param, stream=stream, **hp)

    def cpu_paged(i, stream=None):
        q.qlora_adamw_paged(grad, master_h, m_h, v_h, grad_h, i + 1, param_dev=param, param_host=param_h,
                            stream=stream, **hp)

    def alone(fn):
        ts = []
        for i in range(reps):
            flush_l2(l2)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(i)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.median(ts))

    def beside_step(fn):
        base, over = [], []
        for i in range(reps):
            for with_opt in (False, True):
                flush_l2(l2)
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                eb = torch.cuda.Event()
                e0.record()
                q.qlora_quantize_nf4(wl.w, out=wl.qw)
                q.qlora_linear_fwd(wl.qw, wl.x, wl.a, wl.b, p.alpha, y=wl.y, u=wl.u, ws=wl.ws)
                eb.record()
                if with_opt:
                    side.wait_event(eb)
                    fn(i, stream=side)
                q.qlora_linear_bwd(wl.qw, wl.x, wl.u, wl.dy, wl.a, wl.b, p.alpha, dx=wl.dx, da=wl.da, db=wl.db,
                                   ws=wl.ws)
                if with_opt:
                    torch.cuda.current_stream().wait_stream(side)
                e1.record()
                torch.cuda.synchronize()
                (over if with_opt else base).append(e0.elapsed_time(e1))
        tb, to = float(np.median(base)), float(np.median(over))
        return tb, to

    t_dev = alone(gpu_device_states)
    t_hostk = alone(gpu_host_states)
    t_cpu = alone(cpu_paged)
    tb1, to1 = beside_step(gpu_host_states)
    tb2, to2 = beside_step(cpu_paged)
    return {"params": n,
            "ms_device_states": round(t_dev, 4),
            "gpu_update_host_states": {"ms": round(t_hostk, 4), "host_link_GB/s": round(16.0 * n / (t_hostk * 1e-3) / 1e9, 1),
                                       "step_ms": round(tb1, 4), "step_ms_with_update": round(to1, 4),
                                       "throughput_loss": round(to1 / tb1 - 1.0, 4)},
            "cpu_update_paged": {"ms": round(t_cpu, 4), "cpu_threads": os.cpu_count(),
                                 "step_ms": round(tb2, 4), "step_ms_with_update": round(to2, 4),
                                 "throughput_loss": round(to2 / tb2 - 1.0, 4)},
            "method": "7B-MLP quantize+fwd+bwd on the main stream; the update on a second stream from the start "
                      "of the backward; medians of 10"}


def fused_siblings(q, device, l2, reps=5):
    """7B attention q, k, v (3 x 4096x4096, r = 64 each, 4096 tokens):
    forward + backward as three separate calls vs one call on the weights
    concatenated along d_out, adapters stacked along the rank and B block
    diagonal (x and x A^T streamed once)."""
    k, n, r, m, alpha = 4096, 4096, 64, 4096, 16.0
    ws = [synth.weight(n, k, seed=40 + i).to(device) for i in range(3)]
    As = [synth.lora_a(r, k, seed=50 + i).to(device) for i in range(3)]
    Bs = [synth.lora_b(n, r, seed=60 + i).to(device) for i in range(3)]
    x = synth.tokens(m, k, seed=7).to(device)
    dy = synth.grad_out(m, 3 * n, seed=8).to(device)
    qws = [q.qlora_quantize_nf4(w) for w in ws]
    qc = q.qlora_quantize_nf4(torch.cat(ws, 0))
    a_cat = torch.cat(As, 0)
    b_bd = torch.zeros((3 * n, 3 * r), dtype=torch.bfloat16, device=device)
    for i in range(3):
        b_bd[i * n:(i + 1) * n, i * r:(i + 1) * r] = Bs[i]
    dys = [dy[:, i * n:(i + 1) * n].contiguous() for i in range(3)]
    ws1 = torch.empty(q.qlora_workspace_bytes(m, n, k, r) + 256, dtype=torch.uint8, device=device)
    ws3 = torch.empty(q.qlora_workspace_bytes(m, 3 * n, k, 3 * r) + 256, dtype=torch.uint8, device=device)

    def separate():
        for i in range(3):
            y, u = q.qlora_linear_fwd(qws[i], x, As[i], Bs[i], alpha, ws=ws1)
            q.qlora_linear_bwd(qws[i], x, u, dys[i], As[i], Bs[i], alpha, ws=ws1)

    def fused():
        y, u = q.qlora_linear_fwd(qc, x, a_cat, b_bd, 3 * alpha, ws=ws3)
        q.qlora_linear_bwd(qc, x, u, dy, a_cat, b_bd, 3 * alpha, ws=ws3)

    out = {}
    for name, fn in (("separate", separate), ("fused", fused)):
        fn()
        ts = []
        for _ in range(reps):
            flush_l2(l2)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        out[name + "_ms"] = round(float(np.median(ts)), 4)
    fl = 3 * (fwd_flops(m, n, k, r) + bwd_flops(m, n, k, r))
    out["separate_TFLOP/s"] = round(fl / (out["separate_ms"] * 1e-3) / 1e12, 1)
    out["fused_TFLOP/s"] = round(fl / (out["fused_ms"] * 1e-3) / 1e12, 1)
    out["speedup"] = round(out["separate_ms"] / out["fused_ms"], 3)
    out["workload"] = "7B attention q,k,v: 3 x 4096x4096 NF4, r=64 each, 4096 tokens, fwd+bwd"
    return out


def gemm_schedule(q, device, l2, reps=5):
    """The pair GEMMs' schedule on the 65B-shaped projections (gate/up 22016x8192
    and down 8192x22016, 4096 tokens, r=64): forward + backward under the
    automatic rule (stream-K for these reductions of >= 128 k-tiles) against
    forced data-parallel; median of `reps` calls, L2 flushed before each."""
    out = {}
    for p in (synth.GATE65B, synth.DOWN65B):
        t = synth.make(p, seed=90)
        qw = q.qlora_quantize_nf4(t["w"].to(device))
        x, a, b, dy = (t[k_].to(device) for k_ in ("x", "a", "b", "dy"))
        del t
        y = torch.empty((p.m, p.n), dtype=torch.bfloat16, device=device)
        u = torch.empty((p.m, p.r), dtype=torch.bfloat16, device=device)
        dx = torch.empty((p.m, p.k), dtype=torch.bfloat16, device=device)
        da = torch.empty((p.r, p.k), dtype=torch.float32, device=device)
        db = torch.empty((p.n, p.r), dtype=torch.float32, device=device)
        ws = torch.empty(q.qlora_workspace_bytes(p.m, p.n, p.k, p.r) + 256, dtype=torch.uint8, device=device)
        res = {}
        for name, mode in (("auto", q.SCHED_AUTO), ("data_parallel", q.SCHED_DATA_PARALLEL)):
            q.qlora_set_gemm_schedule(mode)
            try:
                ts = {"fwd": [], "bwd": []}
                for i in range(reps + 2):
                    flush_l2(l2)
                    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                    e[0].record()
                    q.qlora_linear_fwd(qw, x, a, b, p.alpha, y=y, u=u, ws=ws)
                    e[1].record()
                    q.qlora_linear_bwd(qw, x, u, dy, a, b, p.alpha, dx=dx, da=da, db=db, ws=ws)
                    e[2].record()
                    torch.cuda.synchronize()
                    if i >= 2:
                        ts["fwd"].append(e[0].elapsed_time(e[1]))
                        ts["bwd"].append(e[1].elapsed_time(e[2]))
            finally:
                q.qlora_set_gemm_schedule(q.SCHED_AUTO)
            f_ms, b_ms = float(np.median(ts["fwd"])), float(np.median(ts["bwd"]))
            res[name] = {"fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
                         "TFLOP/s": round((fwd_flops(p.m, p.n, p.k, p.r) + bwd_flops(p.m, p.n, p.k, p.r))
                                          / ((f_ms + b_ms) * 1e-3) / 1e12, 1)}
        res["speedup"] = round((res["data_parallel"]["fwd_ms"] + res["data_parallel"]["bwd_ms"])
                               / (res["auto"]["fwd_ms"] + res["auto"]["bwd_ms"]), 3)
        out[p.name] = res
        del qw, x, a, b, dy, y, u, dx, da, db, ws
        torch.cuda.empty_cache()
    return out


def whole_stack(q, device, l2):
    """The whole 7B-shaped stack: 32 layers of q, k, v, o (4096x4096), gate,
    up (11008x4096) and down (4096x11008), 6,476,005,376 weights ~ N(0, 0.02).
    Each weight is generated on the GPU from its own seed; the 224 quantize
    calls (NF4 + double quantization) then run back to back inside one event
    pair, and the bf16 copies are freed. Then forward + backward of all 224
    quantized linears at 4096 tokens with r = 64 adapters, one event pair
    around the whole sweep."""
    m, r, alpha = 4096, 64, 16.0
    lin, ws_bf16, params = [], [], 0
    for layer in range(synth.STACK7B_LAYERS):
        for idx, (_, n, k) in enumerate(synth.STACK7B_LAYER):
            w, a, b = synth.stack_linear(layer, idx, r=r, device=device)
            ws_bf16.append(w)
            lin.append((q.NF4Weight(n, k, device=device), n, k, a, b))
            params += n * k
    # all 224 quantize calls back to back (12.95 GB of bf16 in, resident)
    flush_l2(l2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for w, (qw, _, _, _, _) in zip(ws_bf16, lin):
        q.qlora_quantize_nf4(w, out=qw)
    e1.record()
    torch.cuda.synchronize()
    q_ms = e0.elapsed_time(e1)
    del ws_bf16
    xs, dys = synth.stack_activations(m, device=device)
    ys = {n: torch.empty((m, n), dtype=torch.bfloat16, device=device) for n in (4096, 11008)}
    dxs = {k: torch.empty((m, k), dtype=torch.bfloat16, device=device) for k in (4096, 11008)}
    u = torch.empty((m, r), dtype=torch.bfloat16, device=device)
    das = {k: torch.empty((r, k), dtype=torch.float32, device=device) for k in (4096, 11008)}
    dbs = {n: torch.empty((n, r), dtype=torch.float32, device=device) for n in (4096, 11008)}
    ws = torch.empty(max(q.qlora_workspace_bytes(m, n, k, r) for _, n, k, _, _ in lin) + 256, dtype=torch.uint8,
                     device=device)

    def sweep():
        for qw, n, k, a, b in lin:
            q.qlora_linear_fwd(qw, xs[k], a, b, alpha, y=ys[n], u=u, ws=ws)
            q.qlora_linear_bwd(qw, xs[k], u, dys[n], a, b, alpha, dx=dxs[k], da=das[k], db=dbs[n], ws=ws)

    sweep()
    flush_l2(l2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    sweep()
    e1.record()
    torch.cuda.synchronize()
    t_ms = e0.elapsed_time(e1)
    # the same sweep captured once as a CUDA graph and replayed (no host
    # launch work between the 448 calls)
    side = torch.cuda.Stream(device=device)
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        sweep()
    g.replay()
    torch.cuda.synchronize()
    flush_l2(l2)
    torch.cuda.synchronize()
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    tg_ms = e0.elapsed_time(e1)
    del g
    st, bits = q.qlora_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({bits:#x}) in the stack sweep")
    fl = sum(fwd_flops(m, n, k, r) + bwd_flops(m, n, k, r) for _, n, k, _, _ in lin)
    qb = sum(quant_bytes(n, k) for _, n, k, _, _ in lin)
    fused = stack_fused_siblings(q, lin, xs, m, r, alpha, l2, fl)
    popt = stack_paged_optimizer(q, lin, xs, dys, ys, dxs, ws, m, r, alpha, l2)
    del lin
    return {"weights": params, "linears": 224, "quantize_ms": round(q_ms, 3), "paged_optimizer": popt,
            "fused_siblings": fused,
            "quantize_GB/s": round(qb / (q_ms * 1e-3) / 1e9, 1), "fwd_bwd_ms": round(t_ms, 3),
            "fwd_bwd_TFLOP": round(fl / 1e12, 2), "fwd_bwd_TFLOP/s": round(fl / (t_ms * 1e-3) / 1e12, 1),
            "fwd_bwd_graph_ms": round(tg_ms, 3), "fwd_bwd_graph_TFLOP/s": round(fl / (tg_ms * 1e-3) / 1e12, 1),
            "workload": "whole 7B-shaped stack, 32 x (q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008), "
                        "4096 tokens, r=64, weights generated on the GPU per layer"}


def concat_nf4(q, parts):
    """The packed weight of parts' matrices stacked along d_out: the codes,
    scale codes and group constants concatenate (blocks lie within rows, and
    each part's row count times its blocks per row is a whole number of
    256-block groups), so no re-quantization is needed."""
    n = sum(p.n_out for p in parts)
    out = q.NF4Weight(n, parts[0].k_in, device=parts[0].codes.device)
    for name in ("codes", "scale_codes", "absmax"):
        torch.cat([getattr(p, name) for p in parts], out=getattr(out, name))
    return out


def stack_fused_siblings(q, lin, xs, m, r, alpha, l2, fl):
    """The whole stack's fwd+bwd with sibling projections fused, as a
    deployment would run it: per layer one call for q, k, v (12288 x 4096,
    adapters stacked to r = 192, B block diagonal) and one for gate, up
    (22016 x 4096, r = 128), o and down as before. Same algorithmic FLOPs as
    the 224 separate linears; one event pair around the sweep, L2 flushed
    first."""
    dev = xs[4096].device
    per_layer = len(synth.STACK7B_LAYER)
    groups = []
    for layer in range(synth.STACK7B_LAYERS):
        lp = lin[layer * per_layer:(layer + 1) * per_layer]
        for idx in ((0, 1, 2), (3,), (4, 5), (6,)):
            parts = [lp[i] for i in idx]
            if len(parts) == 1:
                qw, n, k, a, b = parts[0]
                groups.append((qw, n, k, a, b, alpha, r))
                continue
            qc = concat_nf4(q, [p_[0] for p_ in parts])
            n = sum(p_[1] for p_ in parts)
            k = parts[0][2]
            rr = r * len(parts)
            a_cat = torch.cat([p_[3] for p_ in parts], 0)
            b_bd = torch.zeros((n, rr), dtype=torch.bfloat16, device=dev)
            row = 0
            for j, p_ in enumerate(parts):
                b_bd[row:row + p_[1], j * r:(j + 1) * r] = p_[4]
                row += p_[1]
            groups.append((qc, n, k, a_cat, b_bd, alpha * len(parts), rr))
    gen = torch.Generator(device=dev)
    gen.manual_seed(synth.STACK7B_ACT_SEED + 1)
    dys = {n: torch.randn((m, n), generator=gen, device=dev).to(torch.bfloat16) for n in (4096, 11008, 12288, 22016)}
    ys = {n: torch.empty((m, n), dtype=torch.bfloat16, device=dev) for n in dys}
    dxs = {k: torch.empty((m, k), dtype=torch.bfloat16, device=dev) for k in (4096, 11008)}
    us = {rr: torch.empty((m, rr), dtype=torch.bfloat16, device=dev) for rr in (r, 2 * r, 3 * r)}
    das = {(rr, k): torch.empty((rr, k), dtype=torch.float32, device=dev) for rr in (r, 2 * r, 3 * r)
           for k in (4096, 11008)}
    dbs = {(n, rr): torch.empty((n, rr), dtype=torch.float32, device=dev) for n in dys for rr in (r, 2 * r, 3 * r)}
    wsz = max(q.qlora_workspace_bytes(m, n, k, rr) for _, n, k, _, _, _, rr in groups)
    ws = torch.empty(wsz + 256, dtype=torch.uint8, device=dev)

    def sweep():
        for qw, n, k, a, b, al, rr in groups:
            q.qlora_linear_fwd(qw, xs[k], a, b, al, y=ys[n], u=us[rr], ws=ws)
            q.qlora_linear_bwd(qw, xs[k], us[rr], dys[n], a, b, al, dx=dxs[k], da=das[(rr, k)], db=dbs[(n, rr)],
                               ws=ws)

    sweep()
    flush_l2(l2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    sweep()
    e1.record()
    torch.cuda.synchronize()
    t_ms = e0.elapsed_time(e1)
    st, bits = q.qlora_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({bits:#x}) in the fused stack sweep")
    return {"calls": 2 * len(groups), "fwd_bwd_ms": round(t_ms, 3),
            "fwd_bwd_TFLOP/s": round(fl / (t_ms * 1e-3) / 1e12, 1),
            "workload": "the same stack with q,k,v fused (12288x4096, r=192) and gate,up fused (22016x4096, r=128) "
                        "per layer; o and down separate; FLOPs counted as for the separate linears"}


def stack_paged_optimizer(q, lin, xs, dys, ys, dxs, ws, m, r, alpha, l2, steps=3):
    """The optimizer's cost per training step of the whole stack, the unit in
    which the pages quote the paged optimizer's throughput loss. One step is
    the forward of all 224 quantized linears (each saving its u'), then their
    backward in reverse order; as soon as a linear's dA, dB are written, the
    AdamW update of its adapter pair (160,067,584 parameters over the stack)
    is queued on a second stream, so the updates overlap the rest of the
    backward, and the step ends when both streams are done. The update runs
    five ways: none; the GPU kernel with m, v in device memory; the GPU
    kernel with m, v paged out to pinned host memory (read and written over
    the host link by the kernel); the same states paged by the copy engines
    (copied into device staging buffers, updated there, copied back; two
    streams in turn); the CPU update (gradient copied to the host, AdamW on
    the host cores, bf16 adapter copied back). Medians of `steps` steps, L2
    flushed before each."""
    dev = xs[4096].device
    sizes = [r * k + n * r for _, n, k, _, _ in lin]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    total = int(offs[-1])
    param = torch.empty(total, dtype=torch.bfloat16, device=dev)
    grad = torch.zeros(total, dtype=torch.float32, device=dev)
    views = []
    for i, (qw, n, k, a, b) in enumerate(lin):
        o = int(offs[i])
        pa, pb = param[o:o + r * k].view(r, k), param[o + r * k:o + sizes[i]].view(n, r)
        pa.copy_(a)
        pb.copy_(b)
        views.append((pa, pb, grad[o:o + r * k].view(r, k), grad[o + r * k:o + sizes[i]].view(n, r)))
    master = param.float()
    m_d, v_d = torch.zeros(total, device=dev), torch.zeros(total, device=dev)
    m_h, v_h = torch.zeros(total).pin_memory(), torch.zeros(total).pin_memory()
    master_h = param.float().cpu().pin_memory()
    grad_h = torch.empty(total).pin_memory()
    param_h = torch.empty(total, dtype=torch.bfloat16).pin_memory()
    us = [torch.empty((m, r), dtype=torch.bfloat16, device=dev) for _ in lin]
    sides = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]
    most = max(sizes)
    stage = [(torch.empty(most, device=dev), torch.empty(most, device=dev)) for _ in sides]
    hp = dict(lr=1e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0)
    evs = [torch.cuda.Event() for _ in lin]

    def update_fn(kind):
        # (i, t, stream): the update of adapter pair i at step t on `stream`
        def dev_states(i, t, st):
            o, e = int(offs[i]), int(offs[i + 1])
            q.qlora_adamw_step(master[o:e], grad[o:e], m_d[o:e], v_d[o:e], t, param=param[o:e], stream=st, **hp)

        def host_states(i, t, st):
            o, e = int(offs[i]), int(offs[i + 1])
            q.qlora_adamw_step(master[o:e], grad[o:e], m_h[o:e], v_h[o:e], t, param=param[o:e], stream=st, **hp)

        def staged(i, t, st):
            o, e = int(offs[i]), int(offs[i + 1])
            ms, vs = stage[i % 2]
            q.qlora_adamw_staged(master[o:e], grad[o:e], m_h[o:e], v_h[o:e], ms[:e - o], vs[:e - o], t,
                                 param=param[o:e], stream=st, **hp)

        def cpu(i, t, st):
            o, e = int(offs[i]), int(offs[i + 1])
            q.qlora_adamw_paged(grad[o:e], master_h[o:e], m_h[o:e], v_h[o:e], grad_h[o:e], t, param_dev=param[o:e],
                                param_host=param_h[o:e], stream=st, **hp)
        return {"none": None, "gpu_device_states": dev_states, "gpu_host_states": host_states,
                "gpu_staged_states": staged, "cpu_paged": cpu}[kind]

    def step(upd, t, two):
        main = torch.cuda.current_stream()
        for i, (qw, n, k, a, b) in enumerate(lin):
            pa, pb, _, _ = views[i]
            q.qlora_linear_fwd(qw, xs[k], pa, pb, alpha, y=ys[n], u=us[i], ws=ws)
        for i in reversed(range(len(lin))):
            qw, n, k, _, _ = lin[i]
            pa, pb, ga, gb = views[i]
            q.qlora_linear_bwd(qw, xs[k], us[i], dys[n], pa, pb, alpha, dx=dxs[k], da=ga, db=gb, ws=ws)
            if upd is not None:
                st = sides[i % 2] if two else sides[0]
                evs[i].record(main)
                st.wait_event(evs[i])
                upd(i, t, st)
        if upd is not None:
            for st in sides:
                main.wait_stream(st)

    out, t = {}, 0
    for kind in ("none", "gpu_device_states", "gpu_host_states", "gpu_staged_states", "cpu_paged"):
        upd = update_fn(kind)
        two = kind == "gpu_staged_states"    # two streams in turn: H2D and D2H of consecutive updates overlap
        t += 1
        step(upd, t, two)                   # warm-up
        torch.cuda.synchronize()
        times = []
        for _ in range(steps):
            t += 1
            flush_l2(l2)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            step(upd, t, two)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        out[kind] = float(np.median(times))
    st, bits = q.qlora_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({bits:#x}) in the stack training steps")
    base = out["none"]
    res = {"adapter_params": total, "step_ms_no_update": round(base, 3),
           "method": "224 forwards then 224 backwards in reverse; each pair's AdamW queued on a second stream "
                     "when its dA, dB are written; medians of %d steps" % steps}
    for kind in ("gpu_device_states", "gpu_host_states", "gpu_staged_states", "cpu_paged"):
        res[kind] = {"step_ms": round(out[kind], 3), "throughput_loss": round(out[kind] / base - 1.0, 4)}
    res["gpu_host_states"]["host_link_bytes_per_step"] = 16 * total
    res["gpu_staged_states"]["host_link_bytes_per_step"] = 16 * total
    res["cpu_paged"]["cpu_threads"] = os.cpu_count()
    res["pages_quote"] = "about 8% throughput loss for the paged optimizer"
    return res


def cpu_baseline_sample(target_s=15.0):
    """Time the oracle (as it stands) on a bounded sample of the same step:
    quantize the full W, forward + backward for `tok` tokens (fp64)."""
    from oracle import linear, nf4
    p = synth.MLP7B
    t = synth.make(p)
    cores = len(os.sched_getaffinity(0))
    w = t["w"].float().numpy()
    x = t["x"].float().numpy().astype(np.float64)
    a = t["a"].float().numpy().astype(np.float64)
    b = t["b"].float().numpy().astype(np.float64)
    dy = t["dy"].float().numpy().astype(np.float64)
    t0 = time.perf_counter()
    o = nf4.quantize(w)
    w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"]).astype(np.float64)
    t_quant = time.perf_counter() - t0
    tok = 64
    t1 = time.perf_counter()
    linear.forward(x[:tok], w_hat, a, b, p.scale)
    linear.backward(x[:tok], dy[:tok], w_hat, a, b, p.scale)
    t_lin = time.perf_counter() - t1
    # grow the token sample until the linear part takes a few seconds (bounded)
    while t_lin < 0.3 * target_s and tok < p.m:
        tok = min(p.m, tok * 4)
        t1 = time.perf_counter()
        linear.forward(x[:tok], w_hat, a, b, p.scale)
        linear.backward(x[:tok], dy[:tok], w_hat, a, b, p.scale)
        t_lin = time.perf_counter() - t1
    flops = fwd_flops(tok, p.n, p.k, p.r) + bwd_flops(tok, p.n, p.k, p.r)
    # scaled to the step's unit: the full step's FLOPs over (quantize + linear time scaled to 4096 tokens)
    full_time = t_quant + t_lin * (p.m / tok)
    value = (fwd_flops(p.m, p.n, p.k, p.r) + bwd_flops(p.m, p.n, p.k, p.r)) / full_time / 1e12
    return {
        "value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
        "sample": (f"numpy oracle: quantize+restore the full 11008x4096 W ({t_quant:.2f} s), fp64 fwd+bwd on "
                   f"{tok} of 4096 tokens ({t_lin:.2f} s, {flops / 1e9:.1f} GFLOP), scaled to 4096 tokens"),
    }


def oracle_config_timings():
    """The oracle (as it stands) timed on the host cores for every workload,
    each on a bounded sample (a few seconds each), in the unit of its GPU
    figure: the tiny problem in full; the decode call (restore of the full
    4096x4096 weight, then the fp64 forward of one token); the 65B gate/up
    projection's quantizer on 1024 of its 22016 rows and its fp64 fwd+bwd on
    16 tokens over those rows; the whole stack's quantizer on 512 rows of
    each of its seven projection shapes."""
    from oracle import linear, nf4
    cores = len(os.sched_getaffinity(0))
    out = {"cores": cores, "kind": "oracle"}

    def f64(t):
        return t.float().numpy().astype(np.float64)

    def quantize_restore(w):
        o = nf4.quantize(w)
        return nf4.dequantize(o["codes"], o["q2"], o["smax"]).astype(np.float64)

    # tiny: quantize + fwd + bwd in full, repeated for about a second
    p = synth.TINY
    t = synth.make(p)
    w, x, a, b, dy = t["w"].float().numpy(), f64(t["x"]), f64(t["a"]), f64(t["b"]), f64(t["dy"])
    reps, t0 = 0, time.perf_counter()
    while reps < 3 or time.perf_counter() - t0 < 1.0:
        wh = quantize_restore(w)
        linear.forward(x, wh, a, b, p.scale)
        linear.backward(x, dy, wh, a, b, p.scale)
        reps += 1
    dt = (time.perf_counter() - t0) / reps
    out["tiny"] = {"workload": p.name, "us_per_step": round(dt * 1e6, 1),
                   "TFLOP/s": round((fwd_flops(p.m, p.n, p.k, p.r) + bwd_flops(p.m, p.n, p.k, p.r)) / dt / 1e12, 6),
                   "sample": "full problem: quantize, restore, fp64 forward and backward"}
    # decode: restore the whole weight, then one token's forward (the GEMV's bytes per call)
    p = synth.DECODE
    t = synth.make(p)
    t0 = time.perf_counter()
    wh = quantize_restore(t["w"].float().numpy())
    t1 = time.perf_counter()
    linear.forward(f64(t["x"]), wh, f64(t["a"]), f64(t["b"]), p.scale)
    t2 = time.perf_counter()
    out["decode"] = {"workload": p.name, "ms_per_call": round((t2 - t1) * 1e3, 3),
                     "GB/s": round(gemv_bytes(p.n, p.k, p.r) / (t2 - t1) / 1e9, 3),
                     "quantize_restore_s": round(t1 - t0, 3),
                     "sample": "full weight restored once (not timed per call); fp64 forward of one token"}
    # 65B gate/up: quantizer and fwd+bwd on a row sample
    p = synth.GATE65B
    rows = 1024
    w = synth.weight(rows, p.k, seed=0, outliers=True).float().numpy()
    t0 = time.perf_counter()
    wh = quantize_restore(w)
    tq = time.perf_counter() - t0
    tok = 16
    x, a, b, dy = (f64(synth.tokens(tok, p.k)), f64(synth.lora_a(p.r, p.k)), f64(synth.lora_b(rows, p.r)),
                   f64(synth.grad_out(tok, rows)))
    t0 = time.perf_counter()
    linear.forward(x, wh, a, b, p.scale)
    linear.backward(x, dy, wh, a, b, p.scale)
    tl = time.perf_counter() - t0
    out["65b_gate_up"] = {"workload": p.name, "quantize_GB/s": round(quant_bytes(rows, p.k) / tq / 1e9, 4),
                          "fwd_bwd_TFLOP/s": round((fwd_flops(tok, rows, p.k, p.r) + bwd_flops(tok, rows, p.k, p.r))
                                                   / tl / 1e12, 4),
                          "sample": f"{rows} of {p.n} rows quantized and restored; fp64 fwd+bwd of {tok} tokens over those rows"}
    # whole stack: the quantizer on 512 rows of each projection shape
    rows, qb, tq = 512, 0, 0.0
    for idx, (_, n, k) in enumerate(synth.STACK7B_LAYER):
        w = synth.weight(rows, k, seed=idx).float().numpy()
        t0 = time.perf_counter()
        quantize_restore(w)
        tq += time.perf_counter() - t0
        qb += quant_bytes(rows, k)
    out["stack_quantize"] = {"workload": "whole 7B-shaped stack quantizer", "GB/s": round(qb / tq / 1e9, 4),
                             "sample": f"{rows} rows of each of the seven projection shapes (of 6,476,005,376 weights)"}
    return out


def run_ours(args):
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import bit_nf4_quantized_06_b200 as q

    peaks, peaks_src = load_peaks()
    wl = Workload(q, device, rank)
    l2 = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)

    for _ in range(args.warmup):
        wl.step(world)
    torch.cuda.synchronize()
    st, bits = q.qlora_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({bits:#x}) after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = q.qlora_launch_count()
    with ClockSampler(device.index) as clk:
        torch.cuda.nvtx.range_push("timed")     # lets a profiler select exactly the timed steps
        for i in range(args.steps):
            flush_l2(l2)
            wl.step(world, evs[i])
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    launches = q.qlora_launch_count() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    parts = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(args.steps)])
    step_ms_local = float(parts.sum(axis=1).sum()) / args.steps
    step_ms = max_over_ranks(step_ms_local, world)
    st, bits = q.qlora_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} ({bits:#x}) after the timed steps")
    clocks = clk.summary()

    p, d = wl.p, wl.d
    med = np.median(parts, axis=0)
    q_ms, f_ms, b_ms, g_ms = (float(v) for v in med)
    f_fl, b_fl = fwd_flops(p.m, p.n, p.k, p.r), bwd_flops(p.m, p.n, p.k, p.r)
    value = world * wl.flops / (step_ms * 1e-3) / 1e12

    # single-GPU measurements outside the step (N = 1 only: every rank would
    # repeat them on its own GPU)
    extras = world == 1
    if extras:
        merge_ms, mb = merge_timing(q, wl, l2)
        popt = paged_optimizer(q, wl, l2)
        sib = fused_siblings(q, device, l2)
        sched = gemm_schedule(q, device, l2)
        stack = whole_stack(q, device, l2)
        stack["fwd_bwd_frac_of_sustained_bf16"] = round(stack["fwd_bwd_TFLOP/s"] / peaks["bf16_tflops_sustained"], 4)
        stack["quantize_frac_hbm"] = round(stack["quantize_GB/s"] / peaks["hbm_gbs"], 4)
        # decode GEMV steady state + single-call latency
        gemv_ms, gemv_lat_ms, _ = gemv_steady_state(q, device)
        gb = gemv_bytes(d.n, d.k, d.r)
        gemv_gbs = gb / (gemv_ms * 1e-3) / 1e9
        g65_ms, g65_lat_ms, _ = gemv_steady_state(q, device, calls=50, copies=4, d=DECODE65)
        g65_b = gemv_bytes(DECODE65.n, DECODE65.k, DECODE65.r)

    # end to end through host buffers: every step copies its inputs (x, dY,
    # W and the decode input) from pinned host memory and reads its results
    # (dA, dB and the decode output) back; the copies of step i + 1 run on a
    # copy stream into a second set of device buffers while step i computes
    # (the prefetch a training loop's data loader does). The inputs (214 MB
    # per step) are larger than L2, so no flush is needed between steps.
    h2d = (wl.host["x"].numel() + wl.host["dy"].numel() + wl.host["w"].numel()) * 2 + wl.dec_host_x.numel() * 2
    d2h = (wl.da.numel() + wl.db.numel()) * 4 + wl.dy_out.numel() * 2
    e2e_ms = e2e_pipelined(wl, max(3, args.steps // 2), world, h2d, d2h)
    e2e_value = world * wl.flops / (e2e_ms * 1e-3) / 1e12

    peak_t = peaks["bf16_tflops"]
    f_ach = f_fl / (f_ms * 1e-3) / 1e12
    b_ach = b_fl / (b_ms * 1e-3) / 1e12
    q_gbs = quant_bytes(p.n, p.k) / (q_ms * 1e-3) / 1e9
    roof = {
        "bound": "tensor", "kernel": "qlora_linear_fwd (7B-MLP, 4096 tokens: x A^T split-K, reduce, fused restore+GEMM)",
        "achieved": round(f_ach, 1), "peak": peak_t, "unit": "TFLOP/s", "frac": round(f_ach / peak_t, 4),
        "peak_source": f"{peaks_src} bf16 burst", "frac_sustained": round(f_ach / peaks["bf16_tflops_sustained"], 4),
        "traffic": fwd_traffic(), "traffic_source": FWD_TRAFFIC["profile"],
    }
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 (NF4 weights, fp32 accumulate)", "data": "synthetic",
        "config": {"workload": p.name + " fwd+bwd, plus its quantize and a decode GEMV 4096x4096 m=1 r=64",
                   "tokens_per_gpu": p.m, "d_out": p.n, "d_in": p.k, "r": p.r, "alpha": p.alpha,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": "flushed before every step (256 MiB write, outside the timed events)"},
        "parts": {
            "quantize": {"ms": round(q_ms, 4), "GB/s": round(q_gbs, 1), "frac_hbm": round(q_gbs / peaks["hbm_gbs"], 4)},
            "fwd": {"ms": round(f_ms, 4), "TFLOP/s": round(f_ach, 1), "frac": round(f_ach / peak_t, 4)},
            "bwd": {"ms": round(b_ms, 4), "TFLOP/s": round(b_ach, 1), "frac": round(b_ach / peak_t, 4)},
            "decode_in_step": {"ms": round(g_ms, 4)},
        },
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "method": "public API with pinned host inputs and outputs; step i+1's H2D copies on a copy "
                          "stream overlap step i's compute (double-buffered device inputs)"},
        "gpu_launches": int(launches),
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"]},
    }
    if extras:
        line["gemv"] = {"workload": d.name, "us_per_call_steady": round(gemv_ms * 1e3, 3),
                        "us_single_call": round(gemv_lat_ms * 1e3, 3), "bytes_per_call": gb,
                        "GB/s": round(gemv_gbs, 1), "frac_hbm": round(gemv_gbs / peaks["hbm_gbs"], 4),
                        "peak_hbm_gbs": peaks["hbm_gbs"], "frac_vs_8tbs": round(gemv_gbs / 8000.0, 4),
                        "method": "CUDA graph of 200 calls over 32 rotating packed weights (277 MB > 2x L2), x5 replays",
                        "65b_gate": {"workload": DECODE65.name, "us_per_call_steady": round(g65_ms * 1e3, 3),
                                     "us_single_call": round(g65_lat_ms * 1e3, 3), "bytes_per_call": g65_b,
                                     "GB/s": round(g65_b / (g65_ms * 1e-3) / 1e9, 1),
                                     "frac_hbm": round(g65_b / (g65_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                     "method": "CUDA graph of 50 calls over 4 rotating packed weights "
                                               "(367 MB > 2x L2), x5 replays"}}
        line["merge"] = {"workload": p.name + " LoRA merge for export, bf16(W_hat + s B A)", "ms": round(merge_ms, 4),
                         "bytes": int(mb), "GB/s": round(mb / (merge_ms * 1e-3) / 1e9, 1),
                         "frac_hbm": round(mb / (merge_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                         "method": "median of 10 calls, L2 flushed before each"}
        line["paged_optimizer"] = popt
        line["fused_siblings"] = sib
        line["gemm_schedule"] = sched
        line["whole_stack"] = stack
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample()
        line["cpu_baseline_configs"] = oracle_config_timings()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    from oracle import linear, nf4
    p = synth.MLP7B
    t = synth.make(p)
    cores = len(os.sched_getaffinity(0))
    w = t["w"].float().numpy()
    x = t["x"].float().numpy().astype(np.float64)
    a = t["a"].float().numpy().astype(np.float64)
    b = t["b"].float().numpy().astype(np.float64)
    dy = t["dy"].float().numpy().astype(np.float64)

    def step(tok):
        t0 = time.perf_counter()
        o = nf4.quantize(w)
        w_hat = nf4.dequantize(o["codes"], o["q2"], o["smax"]).astype(np.float64)
        t1 = time.perf_counter()
        linear.forward(x[:tok], w_hat, a, b, p.scale)
        linear.backward(x[:tok], dy[:tok], w_hat, a, b, p.scale)
        return t1 - t0, time.perf_counter() - t1

    # Each step is the full quantize + restore and fp64 fwd+bwd on as many of
    # the 4096 tokens as keep the whole run (warm-up and timed steps) within
    # about 150 s on these cores: all of them where the cores allow, so that
    # the step is the GPU arm's workload itself. The first warm-up step
    # measures the rates (256 tokens).
    budget_s = 150.0
    tq0, tf0 = step(256)
    remaining = max(1, args.steps + args.warmup - 1)
    per_tok = tf0 / 256
    tok = int((budget_s / remaining - tq0) / per_tok) // 32 * 32
    tok = max(32, min(p.m, tok))
    for _ in range(args.warmup - 1):
        step(tok)
    tq = tf = 0.0
    for _ in range(args.steps):
        a_, b_ = step(tok)
        tq += a_
        tf += b_
    tq /= args.steps
    tf /= args.steps
    dt = tq + tf
    # the same rate as the GPU arm's: the step's fwd+bwd flops at 4096 tokens
    # over the quantize time plus the fwd+bwd time (scaled to 4096 tokens
    # when fewer were run)
    full = tq + tf * p.m / tok
    value = (fwd_flops(p.m, p.n, p.k, p.r) + bwd_flops(p.m, p.n, p.k, p.r)) / full / 1e12
    if tok == p.m:
        sample = (f"numpy oracle per step: quantize+restore the full 11008x4096 W ({tq:.2f} s), fp64 fwd+bwd on "
                  f"all 4096 tokens ({tf:.2f} s): the GPU arm's step")
        wl = p.name + " fwd+bwd with its quantize (the full step)"
    else:
        sample = (f"numpy oracle per step: quantize+restore the full 11008x4096 W ({tq:.2f} s), fp64 fwd+bwd on "
                  f"{tok} of 4096 tokens ({tf:.2f} s); rate over the step scaled to 4096 tokens ({full:.1f} s)")
        wl = p.name + " fwd+bwd (bounded token sample) with its quantize"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl, "tokens_per_step": tok, "full_step_ms": round(full * 1e3, 1)},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def torchrun_command(n, script, argv, port):
    """The command that starts `n` ranks of `script` on this node, one process
    per GPU (rank i on GPU i through LOCAL_RANK), rendezvous on 127.0.0.1."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), script] + list(argv)


def free_port():
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def spawn_ranks(n, script, argv, timeout_s=1800):
    """Run `script` as `n` ranks under torch.distributed.run and return its exit
    status (the ranks' JSON line is printed by rank 0). Used when the bench is
    started with --gpus N > 1 outside a launcher."""
    cmd = torchrun_command(n, script, argv, free_port())
    return subprocess.call(["timeout", "-k", "60", str(timeout_s)] + cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # data-parallel over N GPUs of this node: start N ranks of this script
        sys.exit(spawn_ranks(args.gpus, os.path.abspath(__file__), sys.argv[1:]))
    if "WORLD_SIZE" in os.environ and int(os.environ["WORLD_SIZE"]) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={os.environ['WORLD_SIZE']}; the run uses WORLD_SIZE",
              file=sys.stderr)
    if args.impl == "reference":
        args.steps = 3 if args.steps is None else args.steps
        args.warmup = 1 if args.warmup is None else args.warmup
        run_reference(args)
    else:
        args.steps = 20 if args.steps is None else args.steps
        args.warmup = 5 if args.warmup is None else args.warmup
        if args.warmup < 3:
            args.warmup = 3
        run_ours(args)


if __name__ == "__main__":
    main()
