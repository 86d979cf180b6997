"""Run a few calls of the denoise-step kernels on one workload, for profilers.

    python tests/profile_case.py [workload] [calls] [e4m3]
    python tests/profile_case.py [workload] [calls] soft_embed [vocab]

Each call is one dd_canvas_attn (dd_canvas_attn_fp8 on the workload's E4M3
inputs with `e4m3`) and one dd_sample_renoise on the workload's step-0
inputs (generated on the GPU), so a profiler that skips the first call of
each kernel sees warm code and a cold-cache second call.  With
`soft_embed`, each call is one dd_soft_embed on the workload's logits and a
synthetic embedding matrix (the vocabulary optionally cut to `vocab` for a
smaller capture).
"""
from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import block_discrete_diffusion_dd_b200 as dd  # noqa: E402
import workloads  # noqa: E402


def main(argv):
    name = argv[1] if len(argv) > 1 else "b1_L4096"
    calls = int(argv[2]) if len(argv) > 2 else 2
    e4m3 = len(argv) > 3 and argv[3] == "e4m3"
    w = workloads.WORKLOADS[name]
    if len(argv) > 3 and argv[3] == "soft_embed":
        if len(argv) > 4:
            w = workloads.scaled(w, vocab=int(argv[4]), name=f"{name}_v{argv[4]}")
        lg = workloads.logits(w, 0, device="cuda")
        E = workloads.embedding(w, device="cuda")
        for _ in range(calls):
            dd.soft_embed(lg, w.temperatures[0], E)
        torch.cuda.synchronize()
        print(f"{w.name} soft_embed: {calls} calls ok")
        return
    if e4m3:
        q, kc, vc, kp, vp, cu, f = workloads.e4m3_attn_inputs(w, 0, device="cuda")
    else:
        q, kc, vc = workloads.canvas_qkv(w, 0, device="cuda")
        kp, vp, cu = workloads.prefix_kv(w, device="cuda")
    lg = workloads.logits(w, 0, device="cuda")
    cud = cu.cuda()
    for i in range(calls):
        if e4m3:
            dd.canvas_attn_fp8(q, kc, vc, kp, vp, cud, f, cu, scale=w.scale)
        else:
            dd.canvas_attn(q, kc, vc, kp, vp, cud, cu, scale=w.scale)
        dd.sample_renoise(lg, w.temperatures[0], w.rates[0], w.seed, i)
    torch.cuda.synchronize()
    print(f"{name}{' e4m3' if e4m3 else ''}: {calls} calls ok")


if __name__ == "__main__":
    main(sys.argv)
