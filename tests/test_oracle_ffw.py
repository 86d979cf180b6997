"""Pins of the oracle's self-conditioning MLP ("DiffusionGemma Technical
Report", paperfeed review, "The mechanism", self-conditioning paragraph:
z_t = FFW(p0 E), a small MLP of 7.8M parameters), read as
z = GELU(u W1 + b1) W2 + b2 with GELU(x) = x Phi(x).

Pinned against: a pure-Python brute force written with math.erf (no
matrix routines, no torch); tabulated values of the standard normal
distribution function; closed forms; linearity in the output layer."""
import math

import numpy as np
import pytest

import oracle
import workloads


def _brute(u, w1, b1, w2, b2):
    rows, d = u.shape
    h = w1.shape[1]
    out = np.zeros((rows, d))
    for r in range(rows):
        hid = []
        for j in range(h):
            a = float(b1[j])
            for k in range(d):
                a += float(u[r, k]) * float(w1[k, j])
            hid.append(a * 0.5 * (1.0 + math.erf(a / math.sqrt(2.0))))
        for c in range(d):
            z = float(b2[c])
            for j in range(h):
                z += hid[j] * float(w2[j, c])
            out[r, c] = z
    return out


def test_ffw_brute_force():
    rng = np.random.default_rng(0)
    u = rng.normal(size=(3, 5)).astype(np.float32)
    w1 = rng.normal(size=(5, 4)).astype(np.float32)
    b1 = rng.normal(size=4).astype(np.float32)
    w2 = rng.normal(size=(4, 5)).astype(np.float32)
    b2 = rng.normal(size=5).astype(np.float32)
    got = oracle.ffw(u, w1, b1, w2, b2)
    want = _brute(u.astype(np.float64), w1.astype(np.float64), b1.astype(np.float64),
                  w2.astype(np.float64), b2.astype(np.float64))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("x,phi", [(0.0, 0.5), (1.0, 0.8413447460685429),
                                   (-1.0, 0.15865525393145707), (2.0, 0.9772498680518208),
                                   (-3.0, 0.0013498980316300946)])
def test_gelu_matches_the_normal_distribution_table(x, phi):
    # one unit through the MLP: W1 = 1, b1 = 0, W2 = 1, b2 = 0 gives GELU(u)
    one = np.ones((1, 1), np.float32)
    z = oracle.ffw(np.full((1, 1), x, np.float32), one, np.zeros(1, np.float32), one,
                   np.zeros(1, np.float32))
    assert z[0, 0] == pytest.approx(x * phi, rel=1e-13, abs=1e-15)


def test_closed_forms_and_linearity():
    rng = np.random.default_rng(1)
    rows, d, h = 4, 8, 6
    u = rng.normal(size=(rows, d)).astype(np.float32)
    w1 = rng.normal(size=(d, h)).astype(np.float32)
    b1 = rng.normal(size=h).astype(np.float32)
    w2 = rng.normal(size=(h, d)).astype(np.float32)
    b2 = rng.normal(size=d).astype(np.float32)
    zero_w1 = np.zeros_like(w1)
    # W1 = 0: every row sees GELU(b1) W2 + b2
    z0 = oracle.ffw(u, zero_w1, b1, w2, b2)
    b64 = b1.astype(np.float64)
    g = b64 * 0.5 * (1 + np.array([math.erf(float(x) / math.sqrt(2)) for x in b64]))
    np.testing.assert_allclose(z0, np.tile(g @ w2.astype(np.float64) + b2.astype(np.float64), (rows, 1)), rtol=1e-12)
    # large positive pre-activations pass through, large negative ones vanish
    big = np.full((1, 1), 40.0, np.float32)
    one = np.ones((1, 1), np.float32)
    zf = np.zeros(1, np.float32)
    assert oracle.ffw(big, one, zf, one, zf)[0, 0] == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.ffw(-big, one, zf, one, zf)[0, 0]) < 1e-300
    # linear in the output layer
    z = oracle.ffw(u, w1, b1, w2, b2)
    z2 = oracle.ffw(u, w1, b1, 2 * w2, 2 * b2)
    np.testing.assert_allclose(z2, 2 * z, rtol=1e-12)
    za = oracle.ffw(u, w1, b1, w2, np.zeros(d, np.float32))
    zb = oracle.ffw(u, w1, b1, w2, np.ones(d, np.float32))
    np.testing.assert_allclose(zb, za + 1.0, rtol=1e-12, atol=1e-12)


def test_self_condition_is_the_mlp_of_the_soft_embedding():
    rng = np.random.default_rng(2)
    rows, V, d, h = 3, 40, 8, 5
    logits = rng.normal(0, 2, (rows, V)).astype(np.float32)
    E = rng.normal(size=(V, d)).astype(np.float32)
    w1 = rng.normal(size=(d, h)).astype(np.float32)
    b1 = rng.normal(size=h).astype(np.float32)
    w2 = rng.normal(size=(h, d)).astype(np.float32)
    b2 = rng.normal(size=d).astype(np.float32)
    z = oracle.self_condition(logits, 0.7, E, w1, b1, w2, b2)
    # softmax written out by hand, then the brute-force MLP
    p = np.exp(logits.astype(np.float64) / 0.7)
    p /= p.sum(axis=1, keepdims=True)
    u = p @ E.astype(np.float64)
    want = _brute(u, w1.astype(np.float64), b1.astype(np.float64), w2.astype(np.float64),
                  b2.astype(np.float64))
    np.testing.assert_allclose(z, want, rtol=1e-11, atol=1e-12)


def test_synthetic_mlp_has_the_pages_parameter_count():
    w = workloads.WORKLOADS["b1_L4096"]
    w1, b1, w2, b2 = workloads.ffw_weights(w)
    n = sum(t.numel() for t in (w1, b1, w2, b2))
    assert round(n / 1e6, 1) == 7.8          # "a small MLP (7.8M parameters)"
    assert w1.shape == (2048, workloads.FFW_HIDDEN) and w2.shape == (workloads.FFW_HIDDEN, 2048)
