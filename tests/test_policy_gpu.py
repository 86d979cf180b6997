"""GPU parity of the pages' sampler policy (dd_entropy_accept,
dd_stop_check, dd_denoise_block_adaptive) against the oracle.

The acceptance and halt decisions are integer outcomes of float64 sums of
float32 entropies; given the same float32 entropies both sides take them
identically, so those comparisons are exact.  The adaptive loop is checked
piece by piece: the same steps driven through the public calls give
bit-identical canvases, and every step's acceptance equals the oracle's on
the entropies the GPU produced; the sampler itself is covered by
test_sampler_gpu.py.
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads

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


def _adaptive_inputs(B=2, S=8, V=8192, L=512, seed=5):
    """Per-step inputs whose logits sharpen step by step, so canvases halt:
    row r carries a spike of height 3 + 4 s at a token fixed per row."""
    w = workloads.scaled(workloads.WORKLOADS["b1_L4096"], batch=B, prefix_lens=(L,) * B,
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
    kp, vp, cu = workloads.prefix_kv(w, device=DEV)
    return w, torch.stack(qs), torch.stack(ks), torch.stack(vs), torch.stack(ls), kp, vp, cu


def test_adaptive_loop_equals_its_pieces_and_the_oracle_rule():
    w, q, kc, vc, lg, kp, vp, cu = _adaptive_inputs()
    S, R, C = q.shape[0], lg.shape[1], 256
    B = R // C
    temps = [oracle.anneal_temperature(s, 48) for s in range(S)]
    budget, thr, seed = 0.1, 0.005, 21
    cud = cu.to(DEV)
    res = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cud, lg, temps, budget, thr, seed,
                                    cu_prefix_host=cu, scale=w.scale)
    n = res["steps_run"]
    assert 1 <= n <= S
    # the same steps through the public calls
    canvas = torch.zeros(R, dtype=torch.int32, device=DEV)
    done = torch.zeros(B, dtype=torch.uint8, device=DEV)
    halt = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    prev = None
    for s in range(n):
        out = dd.sample_renoise(lg[s], temps[s], 0.0, seed, s)
        torch.cuda.synchronize()
        h_gpu, pred = out["entropy"], out["pred"]
        before = done.clone()
        dd.stop_check(h_gpu, pred, prev, C, thr, s, done, halt)
        acc = dd.entropy_accept(h_gpu, pred, C, budget, seed, s, lg.shape[-1])
        ref = oracle.entropy_accept(h_gpu.cpu().numpy(), pred.cpu().numpy(), C, budget, seed, s,
                                    lg.shape[-1])
        for b in range(B):
            sl = slice(b * C, (b + 1) * C)
            if before[b]:
                continue                                   # halted earlier: frozen
            if done[b]:
                canvas[sl] = pred[sl]                      # halts now: its prediction
            else:
                np.testing.assert_array_equal(acc["tokens"][sl].cpu().numpy(), ref["tokens"][sl])
                canvas[sl] = acc["tokens"][sl]
        np.testing.assert_array_equal(res["canvas_history"][s].cpu().numpy(),
                                      canvas.cpu().numpy())
        prev = pred
    np.testing.assert_array_equal(res["halt_step"].cpu().numpy(), halt.cpu().numpy())
    np.testing.assert_array_equal(res["canvas"].cpu().numpy(), canvas.cpu().numpy())
    # the logits sharpen fast enough that every canvas halts before the last step
    assert (res["halt_step"].cpu().numpy() >= 1).all() and n < S


def test_adaptive_graph_replays_the_eager_loop():
    """dd_denoise_block_adaptive_graph: the loop on the device (one IF node
    per step, cleared once every canvas has halted) gives the eager loop's
    canvas, history, halt steps and step count, replay after replay, and
    again after new inputs are written into the captured buffers."""
    w, q, kc, vc, lg, kp, vp, cu = _adaptive_inputs()
    S = q.shape[0]
    temps = [oracle.anneal_temperature(s, 48) for s in range(S)]
    budget, thr, seed = 0.1, 0.005, 21
    cud = cu.to(DEV)
    eager = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cud, lg, temps, budget, thr, seed,
                                      cu_prefix_host=cu, scale=w.scale)
    n = eager["steps_run"]
    assert n < S                                   # halts early: later bodies are skipped
    lb = lg.clone()
    g = dd.denoise_block_adaptive_graph(q, kc, vc, kp, vp, cud, lb, temps, budget, thr, seed,
                                        cu_prefix_host=cu, scale=w.scale)
    for _ in range(2):
        t = g.launch()
        torch.cuda.synchronize()
        assert int(t["steps_run"].item()) == n
        assert torch.equal(t["canvas"], eager["canvas"])
        assert torch.equal(t["halt_step"], eager["halt_step"])
        assert torch.equal(t["canvas_history"][:n], eager["canvas_history"])
    # flatter logits for the first steps: the loop runs longer
    lb[:2].copy_((lg[:2].float() * 0.25).to(torch.bfloat16))
    ref = dd.denoise_block_adaptive(q, kc, vc, kp, vp, cud, lb.clone(), temps, budget, thr, seed,
                                    cu_prefix_host=cu, scale=w.scale)
    t = g.launch()
    torch.cuda.synchronize()
    m = ref["steps_run"]
    assert int(t["steps_run"].item()) == m
    assert torch.equal(t["canvas"], ref["canvas"])
    assert torch.equal(t["halt_step"], ref["halt_step"])
    assert torch.equal(t["canvas_history"][:m], ref["canvas_history"])
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
    g.destroy()
