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


# ------------------------------------------------ the adaptive block loop
# Closed cases for oracle.denoise_block_adaptive, built so that the outcome
# of every step is known without running the loop: a "flat" row (all logits
# equal) has entropy ln V > budget, so it is never accepted and is re-noised
# to its replacement token; a "peaked" row (one logit 60 above the rest) has
# an entropy below 1e-20 and a prediction fixed at its hot token (the Gumbel
# noise lies in [-2.8, 16.7], far below the 60 / tau lead).

V_LOOP, C_LOOP = 64, 8


def _loop_logits(peaked, hot):
    """peaked: bool [S, R]; hot: int [R] -> float32 logits [S, R, V]."""
    S, R = peaked.shape
    lg = np.zeros((S, R, V_LOOP), np.float32)
    for s in range(S):
        for r in range(R):
            if peaked[s, r]:
                lg[s, r, hot[r]] = 60.0
    return lg


def _replacements(lg_s, seed, step):
    # rate 1: every position takes its uniform replacement token (pinned in
    # test_oracle_sampler.py)
    return oracle.sample_renoise(lg_s, 1.0, 1.0, seed, step)["tokens"]


def test_adaptive_loop_halts_at_the_second_stable_low_entropy_step():
    S, k, seed = 6, 3, 17
    hot = np.arange(C_LOOP, dtype=np.int32) * 7 % V_LOOP
    peaked = np.zeros((S, C_LOOP), bool)
    peaked[k - 1:] = True                     # stable from step k-1: halts at step k
    lg = _loop_logits(peaked, hot)
    temps = [oracle.anneal_temperature(s, 48) for s in range(S)]
    r = oracle.denoise_block_adaptive(lg, temps, 0.1, 0.005, seed, C_LOOP)
    assert r["steps_run"] == k + 1 and list(r["halt_step"]) == [k]
    for s in range(k - 1):                    # flat steps: nothing fits the budget
        np.testing.assert_array_equal(r["history"][s], _replacements(lg[s], seed, s))
    np.testing.assert_array_equal(r["history"][k - 1], hot)   # all accepted (entropy ~ 0)
    np.testing.assert_array_equal(r["history"][k], hot)       # halts: its prediction
    np.testing.assert_array_equal(r["canvas"], hot)


def test_adaptive_loop_freezes_a_halted_canvas_and_waits_for_the_others():
    """Canvas 0 halts at step 2, canvas 1 at step 4; canvas 0's logits turn
    flat again after it halted, which must not change it."""
    S, seed = 7, 5
    R = 2 * C_LOOP
    hot = (np.arange(R, dtype=np.int32) * 11 + 3) % V_LOOP
    peaked = np.zeros((S, R), bool)
    peaked[1:3, :C_LOOP] = True               # canvas 0: stable at steps 1, 2 -> halts at 2
    peaked[3:, C_LOOP:] = True                # canvas 1: stable from step 3 -> halts at 4
    lg = _loop_logits(peaked, hot)
    temps = [0.8] * S
    r = oracle.denoise_block_adaptive(lg, temps, 0.1, 0.005, seed, C_LOOP)
    assert r["steps_run"] == 5 and list(r["halt_step"]) == [2, 4]
    c0, c1 = slice(0, C_LOOP), slice(C_LOOP, R)
    np.testing.assert_array_equal(r["history"][0][c0], _replacements(lg[0], seed, 0)[c0])
    for s in range(1, 5):
        np.testing.assert_array_equal(r["history"][s][c0], hot[c0])     # accepted, then frozen
    for s in range(3):
        np.testing.assert_array_equal(r["history"][s][c1], _replacements(lg[s], seed, s)[c1])
    for s in (3, 4):
        np.testing.assert_array_equal(r["history"][s][c1], hot[c1])
    np.testing.assert_array_equal(r["canvas"], hot)


def test_adaptive_loop_without_a_halt_runs_every_step():
    S, seed = 4, 2
    hot = np.arange(C_LOOP, dtype=np.int32) + 40
    peaked = np.ones((S, C_LOOP), bool)
    peaked[:, 5] = False                      # one flat position: mean entropy ln(64) / 8
    lg = _loop_logits(peaked, hot)
    r = oracle.denoise_block_adaptive(lg, [0.8] * S, 0.1, 0.005, seed, C_LOOP)
    assert r["steps_run"] == S and list(r["halt_step"]) == [-1]
    for s in range(S):                        # the 7 peaked positions fit the budget
        want = hot.copy()
        want[5] = _replacements(lg[s], seed, s)[5]
        np.testing.assert_array_equal(r["history"][s], want)
    # a threshold no canvas can meet, on logits that would halt at step 1
    r2 = oracle.denoise_block_adaptive(_loop_logits(np.ones((S, C_LOOP), bool), hot), [0.8] * S,
                                       0.1, -1.0, seed, C_LOOP)
    assert r2["steps_run"] == S and list(r2["halt_step"]) == [-1]
    assert (r2["history"] == hot).all()


def test_adaptive_loop_margins():
    """The margins the GPU tests use to tell near-boundary decisions apart:
    the stop margin is |mean entropy - threshold|; the acceptance margin is
    the distance of the budget to the cut, or the entropy gap at the cut."""
    h = np.array([0.03, 0.01, 0.05, 0.02], np.float32)      # sorted: .01 .02 .03 .05
    # sums .01 .03 .06 | .11 > 0.1: margin = min(0.1 - 0.06, 0.11 - 0.1, 0.05 - 0.03)
    m = oracle._acceptance_margin(h, 0.1)
    want = min(0.1 - (0.01 + 0.02 + 0.03), (0.01 + 0.02 + 0.03 + 0.05) - 0.1, 0.05 - 0.03)
    assert m == pytest.approx(want, abs=1e-7)
    assert oracle._acceptance_margin(np.zeros(4, np.float32), 0.1) == pytest.approx(0.1)
    assert oracle._acceptance_margin(np.full(3, 5.0, np.float32), 0.1) == pytest.approx(4.9)
    S = 2
    hot = np.arange(C_LOOP, dtype=np.int32)
    lg = _loop_logits(np.zeros((S, C_LOOP), bool), hot)
    r = oracle.denoise_block_adaptive(lg, [1.0] * S, 0.1, 0.005, 1, C_LOOP)
    assert r["stop_margin"][0][0] == pytest.approx(np.log(V_LOOP) - 0.005, rel=1e-6)
