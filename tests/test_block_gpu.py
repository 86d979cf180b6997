"""GPU parity of dd_denoise_block (the 12-step inner loop of one block)."""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads
from parity import check_attn, check_sampler

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def block12():
    w = workloads.WORKLOADS["block12_L8192"]
    qs, kcs, vcs, ls = workloads.all_steps(w, device=DEV)
    kp, vp, cu = workloads.prefix_kv(w, device=DEV)
    return w, qs, kcs, vcs, ls, kp, vp, cu


@pytest.fixture(scope="module")
def block12_ref(block12):
    """The oracle's sampler of every step of the 12-step block."""
    w, qs, kcs, vcs, ls, kp, vp, cu = block12
    return [oracle.sample_renoise(ls[s].cpu(), w.temperatures[s], w.rates[s], w.seed, s)
            for s in range(w.steps)]


def test_block12_every_step_matches_oracle(block12, block12_ref):
    w, qs, kcs, vcs, ls, kp, vp, cu = block12
    init = dd.init_canvas(w.rows, w.vocab, w.seed)
    np.testing.assert_array_equal(init.cpu().numpy(), oracle.init_canvas(w.rows, w.vocab, w.seed))
    out = dd.denoise_block(qs, kcs, vcs, kp, vp, cu.to(DEV), ls, w.rates, w.temperatures,
                           seed=w.seed, cu_prefix_host=cu)
    torch.cuda.synchronize()
    hist = out["canvas_history"]
    assert torch.equal(out["canvas"], hist[-1])
    ties = 0
    for s in range(w.steps):
        ref = block12_ref[s]
        got = {"tokens": hist[s], "conf": out["conf_steps"][s]}
        st = check_sampler(got, ref)
        ties += st["near_tie_mismatches"]
    # final canvas (rate 0 at the last step: every position is the sampled id)
    assert w.rates[-1] == 0.0
    print("block12 near-tie mismatches:", ties)
    pos = np.array([0, 100, 255], np.int32)
    for s in (0, 11):
        ref_o, _ = oracle.canvas_attn(qs[s].cpu(), kcs[s].cpu(), vcs[s].cpu(), kp.cpu(), vp.cpu(),
                                      cu.numpy(), w.scale, positions=pos)
        check_attn(out["attn_out"][s], ref_o, torch.bfloat16, positions=pos)


def test_block12_restart_from_step0(block12):
    """Counter-based randomness: restarting at step k reproduces steps k.."""
    w, qs, kcs, vcs, ls, kp, vp, cu = block12
    full = dd.denoise_block(qs, kcs, vcs, kp, vp, cu.to(DEV), ls, w.rates, w.temperatures,
                            seed=w.seed, cu_prefix_host=cu)
    k = 5
    part = dd.denoise_block(qs[k:], kcs[k:], vcs[k:], kp, vp, cu.to(DEV), ls[k:], w.rates[k:],
                            w.temperatures[k:], seed=w.seed, step0=k, cu_prefix_host=cu)
    torch.cuda.synchronize()
    assert torch.equal(part["canvas_history"], full["canvas_history"][k:])
    assert torch.equal(part["conf_steps"], full["conf_steps"][k:])
    assert torch.equal(part["attn_out"], full["attn_out"][k:])


def test_block_without_history_buffers():
    w = workloads.scaled(workloads.WORKLOADS["block12_L8192"], prefix_lens=(300,), vocab=5000,
                         steps=3, rates=(0.9, 0.5, 0.0), temperatures=(1.0, 0.8, 0.6),
                         name="block3")
    qs, kcs, vcs, ls = workloads.all_steps(w, device=DEV)
    kp, vp, cu = workloads.prefix_kv(w, device=DEV)
    out = dd.denoise_block(qs, kcs, vcs, kp, vp, cu.to(DEV), ls, w.rates, w.temperatures,
                           seed=3, cu_prefix_host=cu, keep_history=False)
    torch.cuda.synchronize()
    ref = oracle.sample_renoise(ls[2].cpu(), w.temperatures[2], w.rates[2], 3, 2)
    tok = out["canvas"].cpu().numpy()
    bad = (tok != ref["tokens"]) & (ref["gap"] >= 1e-5)
    assert not bad.any()


def test_block_graph_replays_the_eager_loop(block12, block12_ref):
    """dd_denoise_block_graph: one capture, every replay's steps against the
    oracle, replays identical to the eager loop, including after new inputs
    are written into the captured buffers, and with the launch count of the
    eager loop."""
    w, qs, kcs, vcs, ls, kp, vp, cu = block12
    eager = dd.denoise_block(qs, kcs, vcs, kp, vp, cu.to(DEV), ls, w.rates, w.temperatures,
                             seed=w.seed, cu_prefix_host=cu)
    torch.cuda.synchronize()
    dd.reset_launch_count()
    dd.denoise_block(qs, kcs, vcs, kp, vp, cu.to(DEV), ls, w.rates, w.temperatures,
                     seed=w.seed, cu_prefix_host=cu)
    per_block = dd.launch_count()
    qb, lb = qs.clone(), ls.clone()
    g = dd.denoise_block_graph(qb, kcs, vcs, kp, vp, cu.to(DEV), lb, w.rates, w.temperatures,
                               seed=w.seed, cu_prefix_host=cu)
    torch.cuda.synchronize()
    dd.reset_launch_count()
    for _ in range(2):
        out = g.launch()
        torch.cuda.synchronize()
        for s in range(w.steps):
            check_sampler({"tokens": out["canvas_history"][s], "conf": out["conf_steps"][s]},
                          block12_ref[s])
        assert torch.equal(out["canvas_history"], eager["canvas_history"])
        assert torch.equal(out["conf_steps"], eager["conf_steps"])
        assert torch.equal(out["attn_out"], eager["attn_out"])
    assert dd.launch_count() == 2 * per_block
    # new inputs through the captured buffers: the step-order reversed
    qb.copy_(qs.flip(0))
    lb.copy_(ls.flip(0))
    ref = dd.denoise_block(qs.flip(0).contiguous(), kcs, vcs, kp, vp, cu.to(DEV),
                           ls.flip(0).contiguous(), w.rates, w.temperatures, seed=w.seed,
                           cu_prefix_host=cu)
    out = g.launch()
    torch.cuda.synchronize()
    assert torch.equal(out["canvas_history"], ref["canvas_history"])
    assert torch.equal(out["attn_out"], ref["attn_out"])
    g.destroy()
    dd.query_device_error(g.tensors["workspace"])


def test_block_fp8_matches_the_step_calls_and_the_oracle():
    """dd_denoise_block_fp8: every step identical to dd_canvas_attn_fp8 +
    dd_sample_renoise called one by one; attention within the E4M3 bound of
    the oracle, tokens equal to the oracle's away from near-ties."""
    from test_attn_fp8_gpu import _check
    w = workloads.scaled(workloads.WORKLOADS["block12_L8192"], prefix_lens=(700,), vocab=20000,
                         steps=3, rates=(0.9, 0.4, 0.0), temperatures=(1.0, 0.8, 0.7),
                         name="block3_e4m3")
    qs, kcs, vcs, kp, vp, cu, f = workloads.e4m3_block_inputs(w, device=DEV)
    ls = torch.stack([workloads.logits(w, s, device=DEV) for s in range(w.steps)])
    assert ls.dtype == torch.bfloat16
    out = dd.denoise_block_fp8(qs, kcs, vcs, kp, vp, cu.to(DEV), f, ls, w.rates, w.temperatures,
                               seed=5, cu_prefix_host=cu, scale=w.scale)
    torch.cuda.synchronize()
    assert out["attn_out"].dtype == torch.bfloat16
    assert torch.equal(out["canvas"], out["canvas_history"][-1])
    for s in range(w.steps):
        o, _ = dd.canvas_attn_fp8(qs[s], kcs[s], vcs[s], kp, vp, cu.to(DEV), f[s], cu,
                                  scale=w.scale)
        r = dd.sample_renoise(ls[s], w.temperatures[s], w.rates[s], 5, s)
        torch.cuda.synchronize()
        assert torch.equal(out["attn_out"][s], o)
        assert torch.equal(out["canvas_history"][s], r["tokens"])
        assert torch.equal(out["conf_steps"][s], r["conf"])
        ref = oracle.sample_renoise(ls[s].cpu(), w.temperatures[s], w.rates[s], 5, s)
        check_sampler({"tokens": out["canvas_history"][s], "conf": out["conf_steps"][s]}, ref)
    pos = np.array([0, 77, 255], np.int32)
    for s in (0, 2):
        ref_o, _ = oracle.canvas_attn(qs[s].cpu(), kcs[s].cpu(), vcs[s].cpu(), kp.cpu(), vp.cpu(),
                                      cu.numpy(), w.scale, positions=pos, qkv_scale=f[s])
        _check(out["attn_out"][s], ref_o, vcs[s].cpu(), vp.cpu(), f[s][2], 700 + 256,
               positions=pos)


def test_block_fp8_ragged_batch_without_history():
    """dd_denoise_block_fp8 on two canvases with prefixes 0 and 700 and no
    history buffers: the final canvas equals the last step's one-by-one
    calls (tokens of a rate-0 step are the sampled ids)."""
    w = workloads.scaled(workloads.WORKLOADS["block12_L8192"], batch=2, prefix_lens=(0, 700),
                         vocab=3000, steps=2, rates=(0.6, 0.0), temperatures=(1.0, 0.9),
                         name="block2_e4m3_ragged")
    qs, kcs, vcs, kp, vp, cu, f = workloads.e4m3_block_inputs(w, device=DEV)
    ls = torch.stack([workloads.logits(w, s, device=DEV) for s in range(w.steps)])
    out = dd.denoise_block_fp8(qs, kcs, vcs, kp, vp, cu.to(DEV), f, ls, w.rates, w.temperatures,
                               seed=9, cu_prefix_host=cu, scale=w.scale, keep_history=False)
    o, _ = dd.canvas_attn_fp8(qs[1], kcs[1], vcs[1], kp, vp, cu.to(DEV), f[1], cu, scale=w.scale)
    r = dd.sample_renoise(ls[1], w.temperatures[1], w.rates[1], 9, 1)
    torch.cuda.synchronize()
    assert out["canvas_history"] is None and out["conf_steps"] is None
    assert torch.equal(out["attn_out"][1], o)
    assert torch.equal(out["canvas"], r["tokens"])
