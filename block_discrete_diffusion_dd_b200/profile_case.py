"""Run a few calls of the denoise-step kernels on one workload, for profilers.

    python -m block_discrete_diffusion_dd_b200.profile_case [workload] [calls]

Each call is one dd_canvas_attn and one dd_sample_renoise on the workload's
step-0 inputs (generated on the GPU), so a profiler that skips the first call
of each kernel sees warm code and a cold-cache second call.
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
    w = workloads.WORKLOADS[name]
    q, kc, vc = workloads.canvas_qkv(w, 0, device="cuda")
    kp, vp, cu = workloads.prefix_kv(w, device="cuda")
    lg = workloads.logits(w, 0, device="cuda")
    cud = cu.cuda()
    for i in range(calls):
        dd.canvas_attn(q, kc, vc, kp, vp, cud, cu, scale=w.scale)
        dd.sample_renoise(lg, w.temperatures[0], w.rates[0], w.seed, i)
    torch.cuda.synchronize()
    print(f"{name}: {calls} calls ok")


if __name__ == "__main__":
    main(sys.argv)
