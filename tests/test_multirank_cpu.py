"""The multi-GPU path is replicas only: every rank runs its own canvases with
its own seeds and the process group carries only the barrier and the
max-over-ranks timing.  These tests run that plumbing as two gloo ranks on
the CPU (world size 2), with the rendezvous on 127.0.0.1."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    dist, r, n, _ = bench._dist()
    assert dist.get_backend() == "gloo" and r == rank and n == world
    # the whole-job time is the slowest rank's
    got = bench._max_over_ranks(dist, 1.5 + rank)
    bench._barrier(dist)
    # each rank's replica inputs come from its own seeds
    w = workloads.scaled(workloads.WORKLOADS["tiny_fp32"])
    sets = bench.make_inputs(w, rank, "cpu")
    sig = torch.tensor([float(sets[0]["q"].double().sum()), float(sets[1]["logits"].double().sum())])
    sigs = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(sigs, sig.double())
    out[rank] = (got, [s.tolist() for s in sigs])
    dist.barrier()
    dist.destroy_process_group()


def test_rank_plumbing_on_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as mgr:  # no fork of a threaded process
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        got, sigs = res[rank]
        assert got == 1.5 + (world - 1)                  # max over ranks
        assert sigs[0] != sigs[1]                         # distinct replica inputs
    assert res[0][1] == res[1][1]


def test_reference_arm_under_torchrun_prints_one_line():
    """bench.py --impl reference under torchrun: rank 0 alone runs the oracle
    and prints the JSON line; the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny_fp32"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
