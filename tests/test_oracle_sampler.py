"""Pins for the oracle's sampler, confidence, entropy and re-noise step.

Definitions ("DiffusionGemma Technical Report", paperfeed review): the
sampler works on temperature-scaled logits and per-position entropies ("The
mechanism", sampler paragraph); corruption is to uniformly random vocabulary
tokens (multinomial noise, same section); each token is corrupted
independently with a probability ("Training").  Sampling is Gumbel-max,
whose law is softmax(z / tau).

Pinned against: chi-square tests of the sampled law vs scipy's softmax,
scipy log-softmax / entropy, closed forms (constant logits, a dominant
spike), a binomial test of the re-noise count, chi-square uniformity of the
replacement tokens, and exact invariances (temperature rescaling, row
sharding).
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch


def _broadcast(oracle_mod, z, n_rows, tau=1.0, rate=0.0, seed=0, step=0):
    """n_rows independent draws from one logit row (row stride 0)."""
    row = np.asarray(z, dtype=np.float32)
    return oracle_mod.sample_renoise(row[None, :], tau, rate, seed, step, row_stride=0,
                                     n_rows=n_rows)


@pytest.mark.parametrize("tau", [1.0, 0.7, 2.0])
def test_gumbel_max_law_is_softmax(oracle_mod, tau):
    z = np.array([0.3, -1.2, 1.5, 0.0, 2.1, -0.4], np.float32)
    n = 300_000
    res = _broadcast(oracle_mod, z, n, tau=tau, seed=123, step=4)
    counts = np.bincount(res["pred"], minlength=z.size)
    p = scipy.special.softmax(z.astype(np.float64) / tau)
    assert scipy.stats.chisquare(counts, p * n).pvalue > 1e-3


def test_constant_logits(oracle_mod):
    V, n = 1024, 200_000
    res = _broadcast(oracle_mod, np.full(V, 1.25, np.float32), n, seed=5)
    np.testing.assert_allclose(res["conf"], 1.0 / V, rtol=1e-14)
    np.testing.assert_allclose(res["entropy"], math.log(V), rtol=1e-12)
    counts = np.bincount(res["pred"], minlength=V)
    assert scipy.stats.chisquare(counts).pvalue > 1e-3


def test_dominant_spike_is_always_sampled(oracle_mod):
    """Gumbel noise from 24-bit uniforms lies in [-2.81, 16.64]; a logit 20
    above all others therefore always wins."""
    V, n = 512, 20_000
    z = np.random.default_rng(0).normal(0, 1, V).astype(np.float32)
    z[77] = z.max() + 20.0
    res = _broadcast(oracle_mod, z, n, seed=9)
    assert (res["pred"] == 77).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_conf_entropy_match_scipy(oracle_mod, dtype):
    R, V = 16, 4096
    g = torch.Generator().manual_seed(3)
    logits = (torch.randn((R, V), generator=g) * 3.0).to(dtype)
    tau = 0.8
    res = oracle_mod.sample_renoise(logits, tau, 0.0, 0, 0)
    z = logits.double().numpy() / tau
    lp = scipy.special.log_softmax(z, axis=1)
    np.testing.assert_allclose(res["conf"], np.exp(lp[np.arange(R), res["pred"]]), rtol=1e-12)
    np.testing.assert_allclose(res["entropy"], scipy.stats.entropy(np.exp(lp), axis=1),
                               rtol=1e-12)


def test_renoise_rate_is_binomial(oracle_mod):
    n, V = 200_000, 1000
    for rate in (0.1, 0.3, 0.9):
        res = _broadcast(oracle_mod, np.zeros(V, np.float32), n, rate=rate, seed=21, step=2)
        k = int(res["renoised"].sum())
        assert scipy.stats.binomtest(k, n, float(np.float32(rate))).pvalue > 1e-3


def test_renoise_edge_rates(oracle_mod):
    n, V = 5000, 64
    z = np.random.default_rng(1).normal(0, 1, V).astype(np.float32)
    r0 = _broadcast(oracle_mod, z, n, rate=0.0, seed=1)
    assert r0["renoised"].sum() == 0
    np.testing.assert_array_equal(r0["tokens"], r0["pred"])
    r1 = _broadcast(oracle_mod, z, n, rate=1.0, seed=1)
    assert r1["renoised"].all()
    # re-noise decisions and replacements do not depend on the logits
    r1b = _broadcast(oracle_mod, z * 5, n, rate=1.0, seed=1)
    np.testing.assert_array_equal(r1["tokens"], r1b["tokens"])


def test_tokens_are_pred_or_replacement(oracle_mod):
    n, V = 20_000, 333
    z = np.random.default_rng(2).normal(0, 2, V).astype(np.float32)
    res = _broadcast(oracle_mod, z, n, rate=0.5, seed=4)
    keep = res["renoised"] == 0
    np.testing.assert_array_equal(res["tokens"][keep], res["pred"][keep])
    assert res["tokens"].min() >= 0 and res["tokens"].max() < V


@pytest.mark.parametrize("V,n,bins", [(1024, 200_000, None), (262144, 3000, 32)])
def test_replacements_are_uniform(oracle_mod, V, n, bins):
    """The replacement draw ranges over the whole vocabulary (V = 262144 is
    binned by its top bits to keep the oracle's full-vocabulary pass short)."""
    res = oracle_mod.sample_renoise(np.zeros((1, V), np.float32), 1.0, 1.0, 8, 1, row_stride=0,
                                    n_rows=n)
    t = res["tokens"]
    assert t.min() >= 0 and t.max() < V
    if bins:
        t = t // (V // bins)
    counts = np.bincount(t, minlength=V if bins is None else bins)
    assert scipy.stats.chisquare(counts).pvalue > 1e-3


def test_init_canvas_uniform(oracle_mod):
    V, n = 1024, 200_000
    c = oracle_mod.init_canvas(n, V, 0)
    assert c.min() >= 0 and c.max() < V
    assert scipy.stats.chisquare(np.bincount(c, minlength=V)).pvalue > 1e-3


def test_temperature_rescaling_is_exact(oracle_mod):
    """(c * logits) / (c * tau) == logits / tau exactly for c a power of 2."""
    R, V = 8, 2048
    x = (torch.randn((R, V), generator=torch.Generator().manual_seed(4)) * 2).float()
    a = oracle_mod.sample_renoise(x, 0.5, 0.25, 7, 3)
    b = oracle_mod.sample_renoise(x * 4, 2.0, 0.25, 7, 3)
    for key in ("tokens", "pred", "conf", "entropy", "renoised", "gap"):
        np.testing.assert_array_equal(a[key], b[key])


def test_row_sharding_consistency(oracle_mod):
    """Rows [k, R) computed with row_offset k equal rows k.. of the full call."""
    R, V, k = 12, 1500, 5
    x = (torch.randn((R, V), generator=torch.Generator().manual_seed(5)) * 3).to(torch.bfloat16)
    full = oracle_mod.sample_renoise(x, 1.0, 0.4, 11, 6)
    part = oracle_mod.sample_renoise(x[k:].contiguous(), 1.0, 0.4, 11, 6, row_offset=k)
    sel = oracle_mod.sample_renoise(x, 1.0, 0.4, 11, 6, rows=[k, R - 1])
    for key in ("tokens", "pred", "conf", "entropy", "renoised", "gap"):
        np.testing.assert_array_equal(part[key], full[key][k:])
        np.testing.assert_array_equal(sel[key], full[key][[k, R - 1]])


def test_gap_and_best_consistency(oracle_mod):
    R, V = 64, 4096
    x = (torch.randn((R, V), generator=torch.Generator().manual_seed(6)) * 3).float()
    res = oracle_mod.sample_renoise(x, 1.0, 0.0, 0, 0)
    assert (res["gap"] >= 0).all()
    # the winning score exceeds its own logit by a Gumbel draw in [-2.81, 16.64]
    g = res["best"] - x.double().numpy()[np.arange(R), res["pred"]]
    assert (g > -2.82).all() and (g < 16.65).all()
