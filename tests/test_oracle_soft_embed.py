"""Pins for the oracle's self-conditioning soft embedding (float64).

Definition ("DiffusionGemma Technical Report", paperfeed review, "The
mechanism", self-conditioning paragraph): the previous step's predicted
token distribution p0 = softmax(logits / tau) of each position, pushed
through the embedding matrix E: out[r] = sum_v p0[r, v] E[v].

Pinned against a pure-Python brute force, closed forms, and properties the
definition implies (temperature scaling, linearity in E, row permutation).
"""
import math

import numpy as np
import torch


def _inputs(R, V, d, seed, dtype=torch.float32, lscale=3.0):
    g = torch.Generator().manual_seed(seed)
    lg = (torch.randn((R, V), generator=g) * lscale).to(dtype)
    E = torch.randn((V, d), generator=g).to(dtype)
    return lg, E


def test_brute_force_tiny(oracle_mod):
    lg, E = _inputs(3, 7, 5, seed=1)
    tau = 0.7
    out = oracle_mod.soft_embed(lg, tau, E)
    L, M = lg.tolist(), E.tolist()
    for r in range(3):
        w = [math.exp(x / tau) for x in L[r]]
        tot = sum(w)
        for k in range(5):
            ref = sum(w[v] / tot * M[v][k] for v in range(7))
            assert abs(out[r, k] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_constant_logits_give_the_mean_embedding(oracle_mod):
    V, d = 1000, 16
    _, E = _inputs(1, V, d, seed=2, dtype=torch.bfloat16)
    lg = torch.full((4, V), 1.25).to(torch.bfloat16)
    out = oracle_mod.soft_embed(lg, 0.9, E)
    mean = E.double().mean(0).numpy()
    np.testing.assert_allclose(out, np.broadcast_to(mean, out.shape), rtol=0, atol=1e-13)


def test_one_dominant_logit_selects_its_row(oracle_mod):
    V, d = 512, 8
    lg, E = _inputs(2, V, d, seed=3)
    lg[0, 17] = 2000.0
    lg[1, 400] = 2000.0
    out = oracle_mod.soft_embed(lg, 1.0, E)
    np.testing.assert_allclose(out[0], E[17].double().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[1], E[400].double().numpy(), rtol=0, atol=1e-12)


def test_temperature_scales_the_logits(oracle_mod):
    lg, E = _inputs(5, 300, 12, seed=4)
    a = oracle_mod.soft_embed(lg * 2.0, 2.0, E)
    b = oracle_mod.soft_embed(lg, 1.0, E)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_linear_in_the_embedding_and_row_permutation(oracle_mod):
    lg, E1 = _inputs(6, 200, 10, seed=5)
    _, E2 = _inputs(6, 200, 10, seed=6)
    o1 = oracle_mod.soft_embed(lg, 0.8, E1)
    o2 = oracle_mod.soft_embed(lg, 0.8, E2)
    o12 = oracle_mod.soft_embed(lg, 0.8, (3.0 * E1.double() + E2.double()).float())
    np.testing.assert_allclose(o12, 3.0 * o1 + o2, rtol=0, atol=1e-5)  # E rounded to float32
    perm = np.array([3, 0, 5, 1, 4, 2])
    op = oracle_mod.soft_embed(lg[perm], 0.8, E1)
    np.testing.assert_allclose(op, o1[perm], rtol=0, atol=1e-14)  # BLAS blocking order


def test_subsets_and_chunking_agree(oracle_mod):
    lg, E = _inputs(4, 1000, 9, seed=7, dtype=torch.bfloat16)
    full = oracle_mod.soft_embed(lg, 1.3, E, v_chunk=128)
    part = oracle_mod.soft_embed(lg, 1.3, E, rows=[2, 0], cols=[8, 1, 3], v_chunk=1000)
    np.testing.assert_allclose(part, full[[2, 0]][:, [8, 1, 3]], rtol=0, atol=1e-13)
