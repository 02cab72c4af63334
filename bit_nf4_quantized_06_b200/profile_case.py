"""Run one library call on a named synthetic workload, for profilers.

    python -m bit_nf4_quantized_06_b200.profile_case --op fwd --workload 7b-mlp --iters 3 [--schedule auto|dp|sk]

Ops: quantize, dequantize, fwd (tensor-core path), bwd, gemv (decode path),
merge (LoRA merge for export), adamw (adapter optimizer step, states on device).
Workloads: tiny, decode, 7b-mlp, 65b-gate, 65b-down, decode-65b-gate. The inputs are the
seeded synthetic tensors of ``synth``; every call goes through the C ABI.
Prints one line with the mean device time per call (CUDA events); numbers
printed while running under a profiler are not measurements.
"""

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

import bit_nf4_quantized_06_b200 as q  # noqa: E402

WORKLOADS = {"tiny": synth.TINY, "decode": synth.DECODE, "7b-mlp": synth.MLP7B,
             "65b-gate": synth.GATE65B, "65b-down": synth.DOWN65B,
             "decode-65b-gate": synth.Problem("decode-gemv-22016x8192-m1-r64", 22016, 8192, 1, 64, 16.0,
                                              backward=False)}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["quantize", "dequantize", "fwd", "bwd", "gemv", "merge", "adamw"], required=True)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="7b-mlp")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--schedule", choices=["auto", "dp", "sk"], default="auto",
                    help="GEMM schedule (qlora_set_gemm_schedule): automatic, data-parallel or stream-K")
    a = ap.parse_args(argv)
    q.qlora_set_gemm_schedule({"auto": q.SCHED_AUTO, "dp": q.SCHED_DATA_PARALLEL, "sk": q.SCHED_STREAM_K}[a.schedule])
    p = WORKLOADS[a.workload]
    torch.cuda.set_device(0)
    t = synth.make(synth.Problem(p.name, p.n, p.k, p.m, p.r, p.alpha, p.outliers, True))
    w, x, aa, bb, dy = (t[k].cuda() for k in ("w", "x", "a", "b", "dy"))
    qw = q.qlora_quantize_nf4(w)
    ws = torch.empty(q.qlora_workspace_bytes(p.m, p.n, p.k, p.r) + 256, dtype=torch.uint8, device="cuda")
    y = torch.empty((p.m, p.n), dtype=torch.bfloat16, device="cuda")
    u = torch.empty((p.m, p.r), dtype=torch.bfloat16, device="cuda")
    q.qlora_linear_fwd_ex(qw, x, aa, bb, p.alpha, path=q.FWD_GEMM if p.m > 16 else q.FWD_GEMV, y=y, u=u, ws=ws)
    w_out = torch.empty_like(w)
    na = aa.numel() + bb.numel()
    master = torch.zeros(na, device="cuda")
    grad = torch.full((na,), 1e-3, device="cuda")
    m_st, v_st = torch.zeros(na, device="cuda"), torch.zeros(na, device="cuda")

    def call():
        if a.op == "quantize":
            q.qlora_quantize_nf4(w, out=qw)
        elif a.op == "dequantize":
            q.qlora_dequantize(qw, out=w_out)
        elif a.op == "fwd":
            q.qlora_linear_fwd_ex(qw, x, aa, bb, p.alpha, path=q.FWD_GEMM, y=y, u=u, ws=ws)
        elif a.op == "merge":
            q.qlora_merge_lora(qw, aa, bb, p.alpha, out=w_out)
        elif a.op == "adamw":
            q.qlora_adamw_step(master, grad, m_st, v_st, 1)
        elif a.op == "gemv":
            q.qlora_linear_fwd_ex(qw, x, aa, bb, p.alpha, path=q.FWD_GEMV, y=y, ws=ws, want_u=False)
        else:
            q.qlora_linear_bwd(qw, x, u, dy, aa, bb, p.alpha, ws=ws)

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        call()
    e1.record()
    torch.cuda.synchronize()
    st, bits = q.qlora_device_status()
    if st != 0:
        raise SystemExit(f"device status {st} ({bits:#x})")
    print(f"{a.op} {p.name}: {e0.elapsed_time(e1) / a.iters:.4f} ms/call over {a.iters} calls")


if __name__ == "__main__":
    main()
