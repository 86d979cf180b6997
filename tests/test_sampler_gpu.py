"""GPU parity of dd_sample_renoise / dd_init_canvas against the oracle.

The CUDA sampler streams the logits once and uses an exponential-race prune
before taking logarithms; the oracle evaluates z + g for every entry in
float64.  Both draw the same Philox4x32-10 words.
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads
from parity import check_sampler

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run(logits, tau, rate, seed, step, row_offset=0, **kw):
    out = dd.sample_renoise(logits, tau, rate, seed, step, row_offset, **kw)
    torch.cuda.synchronize()
    return out


def _gen(R, V, std, dtype, seed=0, spike=0.0, device=DEV):
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn((R, V), generator=g, device=device) * std
    if spike:
        idx = torch.randint(0, V, (R,), generator=g, device=device)
        x[torch.arange(R, device=device), idx] += spike
    return x.to(dtype)


def test_tiny_fp32_workload():
    w = workloads.WORKLOADS["tiny_fp32"]
    lg = workloads.logits(w, 0)
    got = _run(lg.to(DEV), w.temperatures[0], w.rates[0], w.seed, 0)
    ref = oracle.sample_renoise(lg, w.temperatures[0], w.rates[0], w.seed, 0)
    st = check_sampler(got, ref)
    print("tiny_fp32", st)


def test_bf16_262k_vocab_all_rows():
    w = workloads.WORKLOADS["b1_L4096"]
    lg = workloads.logits(w, 0, device=DEV)
    got = _run(lg, 1.0, w.rates[0], w.seed, 0)
    ref = oracle.sample_renoise(lg.cpu(), 1.0, w.rates[0], w.seed, 0)
    st = check_sampler(got, ref)
    print("b1_L4096", st)


def test_ragged_b8_rows_sampled():
    """The 2048-row workload in its real launch; 96 rows checked."""
    w = workloads.WORKLOADS["ragged_b8"]
    lg = workloads.logits(w, 0, device=DEV)
    got = _run(lg, 1.0, w.rates[0], w.seed, 0)
    rows = np.unique(np.concatenate([[0, 1, 255, 256, 1023, 2047],
                                     np.random.default_rng(0).integers(0, 2048, 90)]))
    ref = oracle.sample_renoise(lg.cpu(), 1.0, w.rates[0], w.seed, 0, rows=rows)
    st = check_sampler(got, ref, rows=rows)
    print("ragged_b8", st)


@pytest.mark.parametrize("tau", [0.4, 0.8, 1.7])
def test_temperatures(tau):
    lg = _gen(32, 65536, 3.0, torch.bfloat16, seed=1, spike=8.0)
    got = _run(lg, tau, 0.25, 77, 3)
    ref = oracle.sample_renoise(lg.cpu(), tau, 0.25, 77, 3)
    check_sampler(got, ref)


@pytest.mark.parametrize("V", [1, 7, 50001, 1000003])
def test_ragged_vocab_scalar_path(V):
    """V not a multiple of 8: the scalar load path and a ragged last chunk."""
    lg = _gen(8, V, 2.0, torch.float32, seed=V)
    got = _run(lg, 1.0, 0.5, 3, 1)
    ref = oracle.sample_renoise(lg.cpu(), 1.0, 0.5, 3, 1)
    check_sampler(got, ref)
    if V == 1:
        assert (got["pred"].cpu() == 0).all()
        np.testing.assert_allclose(got["conf"].cpu().numpy(), 1.0, rtol=1e-6)
        np.testing.assert_allclose(got["entropy"].cpu().numpy(), 0.0, atol=1e-6)


def test_strided_unaligned_rows():
    base = _gen(16, 20003, 3.0, torch.bfloat16, seed=5)
    lg = base[:, :20000]  # row stride 20003 elements: rows not 16-byte aligned
    got = _run(lg, 1.0, 0.3, 9, 2)
    ref = oracle.sample_renoise(base.cpu(), 1.0, 0.3, 9, 2, vocab=20000, row_stride=20003)
    check_sampler(got, ref)


def test_row_offset_and_shards_agree():
    lg = _gen(64, 8192, 3.0, torch.bfloat16, seed=6)
    full = _run(lg, 1.0, 0.5, 11, 4)
    lo = _run(lg[:40], 1.0, 0.5, 11, 4, row_offset=0)
    hi = _run(lg[40:], 1.0, 0.5, 11, 4, row_offset=40)
    for k in ("tokens", "pred", "conf", "entropy", "renoised"):
        assert torch.equal(torch.cat([lo[k], hi[k]]), full[k])
    ref = oracle.sample_renoise(lg[40:].cpu(), 1.0, 0.5, 11, 4, row_offset=40)
    check_sampler(hi, ref)


@pytest.mark.parametrize("rate", [0.0, 1.0])
def test_edge_rates(rate):
    lg = _gen(128, 4096, 2.0, torch.float32, seed=7)
    got = _run(lg, 1.0, rate, 1, 0)
    ref = oracle.sample_renoise(lg.cpu(), 1.0, rate, 1, 0)
    check_sampler(got, ref)
    assert int(got["renoised"].sum()) == (128 if rate == 1.0 else 0)


def test_constant_logits_closed_form():
    V = 262144
    lg = torch.full((8, V), 0.5, dtype=torch.bfloat16, device=DEV)
    got = _run(lg, 1.0, 0.0, 0, 0)
    np.testing.assert_allclose(got["conf"].cpu().numpy(), 1.0 / V, rtol=1e-5)
    np.testing.assert_allclose(got["entropy"].cpu().numpy(), np.log(V), rtol=1e-5)


def test_deterministic_across_calls():
    lg = _gen(256, 262144, 3.0, torch.bfloat16, seed=8, spike=8.0)
    a = _run(lg, 1.0, 0.3, 5, 9)
    b = _run(lg, 1.0, 0.3, 5, 9)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_workspace_reuse_leaves_state_clear():
    """The sampler keeps a work counter and per-row maxima in the workspace
    and clears them at the end of every call: calls that share one workspace
    (different rows, vocabularies, seeds) give what fresh workspaces give."""
    a_lg = _gen(256, 262144, 3.0, torch.bfloat16, seed=21, spike=8.0)
    b_lg = _gen(40, 50000, 2.0, torch.float32, seed=22)
    ws = dd.new_workspace(max(dd.sample_workspace_bytes(256, 262144),
                              dd.sample_workspace_bytes(40, 50000)))
    a1 = _run(a_lg, 1.0, 0.3, 3, 4, workspace=ws)
    b1 = _run(b_lg, 0.7, 0.5, 4, 5, workspace=ws)
    a2 = _run(a_lg, 1.0, 0.3, 3, 4, workspace=ws)
    b_fresh = _run(b_lg, 0.7, 0.5, 4, 5)
    for k in a1:
        assert torch.equal(a1[k], a2[k]), k
        assert torch.equal(b1[k], b_fresh[k]), k
    check_sampler(b1, oracle.sample_renoise(b_lg.cpu(), 0.7, 0.5, 4, 5))


def test_workspace_shared_across_row_counts_with_negative_logits():
    """A call with fewer rows lays its chunk records over the row maxima of
    a call with more rows; the records are cleared at the end of every call,
    so a later call whose best scores are all far below zero still starts
    from a clear state (a leftover value would outrank every real score)."""
    few = _gen(40, 50000, 2.0, torch.float32, seed=31)
    neg = (_gen(256, 8192, 1.0, torch.float32, seed=32) - 40.0).contiguous()
    ws = dd.new_workspace(max(dd.sample_workspace_bytes(40, 50000, torch.float32),
                              dd.sample_workspace_bytes(256, 8192, torch.float32)))
    _run(few, 1.0, 0.5, 1, 2, workspace=ws)
    got = _run(neg, 1.0, 0.0, 3, 4, workspace=ws)
    dd.query_device_error(ws)
    fresh = _run(neg, 1.0, 0.0, 3, 4)
    for k in got:
        assert torch.equal(got[k], fresh[k]), k
    check_sampler(got, oracle.sample_renoise(neg.cpu(), 1.0, 0.0, 3, 4))


def test_large_seed_and_step():
    lg = _gen(16, 4096, 3.0, torch.bfloat16, seed=9)
    seed, step = 0xDEADBEEFCAFEF00D, 0xFFFFFFF0
    got = _run(lg, 1.0, 0.5, seed, step, row_offset=0xFFFF0000)
    ref = oracle.sample_renoise(lg.cpu(), 1.0, 0.5, seed, step, row_offset=0xFFFF0000)
    check_sampler(got, ref)


def test_init_canvas_matches_oracle():
    for rows, V, seed, off in [(256, 262144, 0, 0), (2048, 1024, 12345, 77), (1, 3, 1, 5)]:
        got = dd.init_canvas(rows, V, seed, off).cpu().numpy()
        np.testing.assert_array_equal(got, oracle.init_canvas(rows, V, seed, off))


def test_launches_are_counted():
    lg = _gen(4, 1024, 1.0, torch.float32)
    dd.reset_launch_count()
    _run(lg, 1.0, 0.5, 0, 0)
    assert dd.launch_count() == 2
