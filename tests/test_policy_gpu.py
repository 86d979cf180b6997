"""GPU parity of the pages' sampler policy (dd_entropy_accept,
dd_stop_check, dd_denoise_block_adaptive) against the oracle.

The acceptance and halt decisions are integer outcomes of float64 sums of
float32 entropies; given the same float32 entropies both sides take them
identically, so the kernel-level comparisons are exact.  The adaptive loop
(eager and on-device graph forms) is compared with the oracle's own loop,
which runs the oracle sampler on the same logits: every step's canvas, the
halt steps and the step count.  No CUDA output enters the oracle.  A canvas
whose decision at some step lies within 1e-5 of its boundary (a Gumbel
near-tie, the halt threshold, the acceptance cut) would be counted and
reported, as for the sampler's near-ties; the inputs here have none.
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads
from parity import check_attn

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _entropies(rng, n):
    # mostly confident positions, some uncertain ones, a few exact ties
    h = np.where(rng.random(n) < 0.75, rng.exponential(2e-3, n), rng.exponential(1.5, n))
    h[rng.integers(0, n, n // 16)] = 0.0125
    return h.astype(np.float32)


@pytest.mark.parametrize("B,C,budget", [(8, 256, 0.1), (3, 256, 0.01), (2, 1024, 0.5),
                                        (5, 100, 0.1), (4, 1, 0.1), (2, 33, 1e9), (2, 64, -1.0)])
def test_entropy_accept_matches_oracle(B, C, budget):
    rng = np.random.default_rng(B * 1000 + C)
    V = 262144
    h = _entropies(rng, B * C)
    pred = rng.integers(0, V, B * C).astype(np.int32)
    got = dd.entropy_accept(torch.from_numpy(h).to(DEV), torch.from_numpy(pred).to(DEV), C,
                            budget, seed=11, step=4, vocab=V, row_offset=7)
    ref = oracle.entropy_accept(h, pred, C, budget, seed=11, step=4, vocab=V, row_offset=7)
    np.testing.assert_array_equal(got["accepted"].cpu().numpy(), ref["accepted"])
    np.testing.assert_array_equal(got["tokens"].cpu().numpy(), ref["tokens"])


def test_stop_check_matches_oracle():
    rng = np.random.default_rng(3)
    B, C = 6, 256
    pred = rng.integers(0, 1000, B * C).astype(np.int32)
    prev = pred.copy()
    prev[1 * C + 17] += 1                        # canvas 1 not stable
    h = np.full(B * C, 1e-3, np.float32)
    h[2 * C:3 * C] = 0.02                        # canvas 2 too uncertain
    h[3 * C:4 * C] = np.float32(2.0 ** -8)       # canvas 3 exactly at a 2^-8 threshold
    done = torch.zeros(B, dtype=torch.uint8, device=DEV)
    done[5] = 1                                  # canvas 5 halted before
    halt = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    dd.stop_check(torch.from_numpy(h).to(DEV), torch.from_numpy(pred).to(DEV),
                  torch.from_numpy(prev).to(DEV), C, 2.0 ** -8, 9, done, halt)
    ref = oracle.stop_check(h, pred, prev, C, 2.0 ** -8)
    got = done.cpu().numpy()
    np.testing.assert_array_equal(got[:5], ref[:5])
    assert got[5] == 1 and halt[5].item() == -7
    assert list(halt[:5].cpu().numpy()) == [9 if ref[b] else -7 for b in range(5)]
    # no previous step: never halts
    done2 = torch.zeros(B, dtype=torch.uint8, device=DEV)
    dd.stop_check(torch.from_numpy(h).to(DEV), torch.from_numpy(pred).to(DEV), None, C, 1.0, 0,
                  done2, halt)
    assert done2.sum().item() == 0


def _adaptive_inputs(B=2, S=8, V=8192, L=512, seed=5, workload="b1_L4096"):
    """Per-step inputs whose logits sharpen step by step, so canvases halt:
    row r carries a spike of height 3 + 4 s at a token fixed per row."""
    w = workloads.scaled(workloads.WORKLOADS[workload], batch=B, prefix_lens=(L,) * B,
                         vocab=V, steps=S, seed=seed)
    g = torch.Generator(device=DEV).manual_seed(seed)
    R = B * 256
    qs, ks, vs, ls = [], [], [], []
    hot = torch.randint(0, V, (R,), generator=g, device=DEV)
    for s in range(S):
        q, kc, vc = workloads.canvas_qkv(w, s, device=DEV)
        lg = torch.randn((R, V), generator=g, device=DEV) * 1.5
        lg[torch.arange(R, device=DEV), hot] += 3.0 + 4.0 * s
        qs.append(q), ks.append(kc), vs.append(vc), ls.append(lg.to(torch.bfloat16))
        del lg
    kp, vp, cu = workloads.prefix_kv(w, device=DEV)
    return w, torch.stack(qs), torch.stack(ks), torch.stack(vs), torch.stack(ls), kp, vp, cu


NEAR = 1e-5  # a decision this close to its boundary may flip with float32 entropies


def _compare_with_oracle(history, halt_step, steps_run, ref, C):
    """Step by step against oracle.denoise_block_adaptive.  A canvas whose
    decision at some step lies within NEAR of its boundary (a top-two Gumbel
    gap, the halt threshold, or the acceptance cut; the oracle reports the
    margins) is counted and left out from that step on, as a near-tie; every
    other canvas must match exactly at every step.  Returns the count."""
    hist = history.cpu().numpy()
    halt = halt_step.cpu().numpy()
    B = halt.size
    live = np.ones(B, bool)
    near = 0
    for s in range(ref["steps_run"]):
        for b in range(B):
            if live[b] and min(ref["min_gap"][s][b], ref["stop_margin"][s][b],
                               ref["accept_margin"][s][b]) < NEAR:
                live[b] = False
                near += 1
        if s >= steps_run:
            break
        for b in np.flatnonzero(live):
            sl = slice(b * C, (b + 1) * C)
            np.testing.assert_array_equal(hist[s][sl], ref["history"][s][sl],
                                          err_msg=f"step {s} canvas {b}")
    for b in np.flatnonzero(live):
        assert halt[b] == ref["halt_step"][b], f"canvas {b} halt step"
    if live.all():
        assert steps_run == ref["steps_run"]
    print(f"adaptive loop: {ref['steps_run']} steps, halt steps {list(ref['halt_step'])}, "
          f"near-boundary canvases {near}")
    return near


def _oracle_loop(lg, temps, budget, thr, seed, C):
    return oracle.denoise_block_adaptive([lg[s].cpu() for s in range(lg.shape[0])], temps,
                                         budget, thr, seed, C)


def test_adaptive_loop_matches_the_oracle():
    """dd_denoise_block_adaptive against oracle.denoise_block_adaptive on two
    canvases: every step's canvas, the halt steps and the step count; the
    attention outputs of the first and last step run at sampled positions."""
    w, q, kc, vc, lg, kp, vp, cu = _adaptive_inputs()
    S, R, C = q.shape[0], lg.shape[1], 256
    temps = [oracle.anneal_temperature(s, 48) for s in range(S)]
    budget, thr, seed = 0.1, 0.005, 21
    attn_out = torch.empty_like(q)
    res = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cu.to(DEV), lg, temps, budget, thr, seed,
                                    cu_prefix_host=cu, scale=w.scale, attn_out=attn_out)
    torch.cuda.synchronize()
    n = res["steps_run"]
    ref = _oracle_loop(lg, temps, budget, thr, seed, C)
    assert _compare_with_oracle(res["canvas_history"], res["halt_step"], n, ref, C) == 0
    np.testing.assert_array_equal(res["canvas"].cpu().numpy(), ref["canvas"])
    # the logits sharpen fast enough that every canvas halts before the last step
    assert (ref["halt_step"] >= 1).all() and ref["steps_run"] < S
    pos = np.array([0, 131, 255], np.int32)
    for s in (0, n - 1):
        ref_o, _ = oracle.canvas_attn(q[s].cpu(), kc[s].cpu(), vc[s].cpu(), kp.cpu(), vp.cpu(),
                                      cu.numpy(), w.scale, positions=pos)
        check_attn(attn_out[s], ref_o, torch.bfloat16, positions=pos)


def test_adaptive_loop_policy_geometry_matches_the_oracle():
    """The pages' policy on the 12-step geometry (one canvas, prefix 8192,
    vocabulary 262144, temperatures annealed 0.8 -> 0.4 over 48 nominal
    steps): the eager loop and its on-device graph form, both against the
    oracle loop, step by step."""
    w, q, kc, vc, lg, kp, vp, cu = _adaptive_inputs(B=1, S=12, V=262144, L=8192, seed=0,
                                                    workload="block12_L8192")
    S, C = q.shape[0], 256
    temps = [oracle.anneal_temperature(s, 48) for s in range(S)]
    budget, thr, seed = 0.1, 0.005, w.seed
    cud = cu.to(DEV)
    res = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cud, lg, temps, budget, thr, seed,
                                    cu_prefix_host=cu, scale=w.scale)
    torch.cuda.synchronize()
    ref = _oracle_loop(lg, temps, budget, thr, seed, C)
    assert 1 <= ref["steps_run"] < S
    assert _compare_with_oracle(res["canvas_history"], res["halt_step"], res["steps_run"], ref,
                                C) == 0
    g = dd.denoise_block_adaptive_graph(q, kc, vc, kp, vp, cud, lg, temps, budget, thr, seed,
                                        cu_prefix_host=cu, scale=w.scale)
    t = g.launch()
    torch.cuda.synchronize()
    m = int(t["steps_run"].item())
    assert _compare_with_oracle(t["canvas_history"][:m], t["halt_step"], m, ref, C) == 0
    np.testing.assert_array_equal(t["canvas"].cpu().numpy(), ref["canvas"])
    g.destroy()
    dd.query_device_error(t["workspace"])


def test_adaptive_graph_matches_the_oracle_replay_after_replay():
    """dd_denoise_block_adaptive_graph: the loop on the device (one IF node
    per step, cleared once every canvas has halted) against the oracle loop,
    replay after replay, and again after new inputs are written into the
    captured buffers."""
    w, q, kc, vc, lg, kp, vp, cu = _adaptive_inputs()
    S, C = q.shape[0], 256
    temps = [oracle.anneal_temperature(s, 48) for s in range(S)]
    budget, thr, seed = 0.1, 0.005, 21
    cud = cu.to(DEV)
    ref = _oracle_loop(lg, temps, budget, thr, seed, C)
    assert ref["steps_run"] < S                     # halts early: later bodies are skipped
    lb = lg.clone()
    g = dd.denoise_block_adaptive_graph(q, kc, vc, kp, vp, cud, lb, temps, budget, thr, seed,
                                        cu_prefix_host=cu, scale=w.scale)
    for _ in range(2):
        t = g.launch()
        torch.cuda.synchronize()
        n = int(t["steps_run"].item())
        assert _compare_with_oracle(t["canvas_history"][:n], t["halt_step"], n, ref, C) == 0
        np.testing.assert_array_equal(t["canvas"].cpu().numpy(), ref["canvas"])
    # flatter logits for the first steps: the loop runs longer
    lb[:2].copy_((lg[:2].float() * 0.25).to(torch.bfloat16))
    ref2 = _oracle_loop(lb, temps, budget, thr, seed, C)
    t = g.launch()
    torch.cuda.synchronize()
    m = int(t["steps_run"].item())
    assert _compare_with_oracle(t["canvas_history"][:m], t["halt_step"], m, ref2, C) == 0
    # the eager loop on the same inputs gives the same bits as the graph
    eager = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cud, lb.clone(), temps, budget, thr,
                                      seed, cu_prefix_host=cu, scale=w.scale)
    assert eager["steps_run"] == m
    assert torch.equal(t["canvas_history"][:m], eager["canvas_history"])
    assert torch.equal(t["halt_step"], eager["halt_step"])
    g.destroy()
    dd.query_device_error(t["workspace"])


def test_adaptive_graph_with_no_halt_runs_every_step():
    """A threshold no canvas meets: every body runs; steps_run = max_steps."""
    w, q, kc, vc, lg, kp, vp, cu = _adaptive_inputs(B=1, S=3)
    temps = [0.8, 0.7, 0.6]
    eager = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cu.to(DEV), lg, temps, 0.1, -1.0, 4,
                                      cu_prefix_host=cu, scale=w.scale)
    assert eager["steps_run"] == 3
    g = dd.denoise_block_adaptive_graph(q, kc, vc, kp, vp, cu.to(DEV), lg, temps, 0.1, -1.0, 4,
                                        cu_prefix_host=cu, scale=w.scale)
    t = g.launch()
    torch.cuda.synchronize()
    assert int(t["steps_run"].item()) == 3
    assert torch.equal(t["canvas_history"], eager["canvas_history"])
    assert t["halt_step"].tolist() == [-1]
    ref = _oracle_loop(lg, temps, 0.1, -1.0, 4, 256)
    assert ref["steps_run"] == 3
    assert _compare_with_oracle(t["canvas_history"], t["halt_step"], 3, ref, 256) == 0
    g.destroy()
