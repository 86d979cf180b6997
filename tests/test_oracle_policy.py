"""Pins of the oracle's sampler policy from the pages ("DiffusionGemma
Technical Report", paperfeed review, "The mechanism", sampler paragraph):
temperature annealed 0.8 -> 0.4, greedy entropy-budget acceptance with
re-noise of the rest, early halt on low mean entropy with a stable
prediction.

The acceptance rule is pinned by the properties that define a greedy
budgeted prefix (they determine the accepted set uniquely), by closed forms,
and by the replacement tokens of the already pinned re-noise rule.
"""
import numpy as np
import pytest

import oracle


def _check_budget_properties(h, acc, budget):
    """Greedy acceptance from lowest entropy: accepted = a prefix of the
    (entropy, position) order whose float64 sum fits the budget, and the next
    position in that order would not fit."""
    h64 = h.astype(np.float64)
    order = sorted(range(h.size), key=lambda i: (h[i], i))
    k = int(acc.sum())
    assert set(np.flatnonzero(acc)) == set(order[:k])          # a prefix of the order
    s = 0.0
    for i in order[:k]:
        s += h64[i]
    assert s <= budget                                           # the budget holds
    if k < h.size:
        assert not (s + h64[order[k]] <= budget)                 # and is maximal
    if 0 < k < h.size:                                           # threshold structure
        assert h[acc == 1].max() <= h[acc == 0].min()


@pytest.mark.parametrize("seed", range(6))
def test_acceptance_is_the_greedy_budgeted_prefix(seed):
    rng = np.random.default_rng(seed)
    C, B = 256, 4
    # mostly confident positions (tiny entropies) plus some uncertain ones
    h = np.where(rng.random(B * C) < 0.7, rng.exponential(1e-3, B * C),
                 rng.exponential(2.0, B * C)).astype(np.float32)
    pred = rng.integers(0, 1000, B * C).astype(np.int32)
    budget = [0.1, 0.01, 0.5, 2.0][seed % 4]
    r = oracle.entropy_accept(h, pred, C, budget, seed=3, step=seed, vocab=1000)
    for b in range(B):
        sl = slice(b * C, (b + 1) * C)
        _check_budget_properties(h[sl], r["accepted"][sl], budget)
        assert r["n_accepted"][b] == r["accepted"][sl].sum()
        assert r["sum_accepted"][b] == pytest.approx(float(h[sl][r["accepted"][sl] == 1]
                                                          .astype(np.float64).sum()), rel=1e-15)


def test_ties_go_to_the_lower_position():
    C = 10
    h = np.full(C, 0.03, np.float32)           # every position equal
    r = oracle.entropy_accept(h, np.arange(C), C, 0.1, 0, 0, 50)
    # 3 * 0.03 fits, 4 * 0.03 does not (float32 0.03 > 0.03)
    assert list(r["accepted"]) == [1, 1, 1] + [0] * 7


def test_closed_forms():
    C = 16
    pred = np.arange(C, dtype=np.int32) + 100
    zero = np.zeros(C, np.float32)
    r = oracle.entropy_accept(zero, pred, C, 0.0, 1, 2, 4096)
    assert r["accepted"].all() and (r["tokens"] == pred).all()      # zero entropy fits b = 0
    h = np.linspace(0.01, 0.5, C).astype(np.float32)
    assert oracle.entropy_accept(h, pred, C, np.inf, 1, 2, 4096)["accepted"].all()
    assert not oracle.entropy_accept(h, pred, C, -1.0, 1, 2, 4096)["accepted"].any()
    # one position far below the rest: exactly that one is accepted
    h2 = np.full(C, 5.0, np.float32)
    h2[7] = 0.05
    r2 = oracle.entropy_accept(h2, pred, C, 0.1, 1, 2, 4096)
    assert list(np.flatnonzero(r2["accepted"])) == [7]


def test_rejected_positions_take_the_replacement_token():
    """Re-noised positions carry the same uniform replacement token as the
    scheduled-rate rule (pinned in test_oracle_sampler.py): with rate 1 every
    position of sample_renoise is replaced."""
    rng = np.random.default_rng(5)
    R, V = 64, 1024
    logits = rng.normal(0, 2, (R, V)).astype(np.float32)
    full = oracle.sample_renoise(logits, 1.0, 1.0, 7, 3)
    h = rng.exponential(0.05, R).astype(np.float32)
    pred = rng.integers(0, V, R).astype(np.int32)
    r = oracle.entropy_accept(h, pred, 32, 0.1, seed=7, step=3, vocab=V)
    acc = r["accepted"] == 1
    assert (r["tokens"][acc] == pred[acc]).all()
    assert (r["tokens"][~acc] == full["tokens"][~acc]).all()


def test_stop_check():
    C = 8
    pred = np.arange(2 * C, dtype=np.int32)
    low = np.full(2 * C, 0.001, np.float32)
    assert list(oracle.stop_check(low, pred, pred, C)) == [1, 1]
    assert list(oracle.stop_check(low, pred, None, C)) == [0, 0]    # no previous step
    moved = pred.copy()
    moved[C + 3] += 1                                                # canvas 1 changed
    assert list(oracle.stop_check(low, moved, pred, C)) == [1, 0]
    at = np.full(C, 2.0 ** -7, np.float32)                          # mean exactly at the threshold
    assert oracle.stop_check(at, pred[:C], pred[:C], C, 2.0 ** -7)[0] == 0     # strict: not below
    assert oracle.stop_check(at, pred[:C], pred[:C], C, 2.0 ** -7 + 1e-12)[0] == 1
    assert oracle.stop_check(np.full(C, 0.0051, np.float32), pred[:C], pred[:C], C)[0] == 0


def test_anneal_schedule():
    S = 48
    t = [oracle.anneal_temperature(s, S) for s in range(S)]
    assert t[0] == pytest.approx(0.8) and t[-1] == pytest.approx(0.4)
    assert all(a > b for a, b in zip(t, t[1:]))                      # strictly decreasing
    assert np.allclose(np.diff(t), -0.4 / 47, atol=1e-7)            # linear
    assert oracle.anneal_temperature(0, 1) == pytest.approx(0.8)
