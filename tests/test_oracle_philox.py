"""Pins for the oracle's Philox4x32-10 and its uniform mapping.

The oracle's generator is written from Salmon et al., "Parallel random
numbers: as easy as 1, 2, 3" (SC'11).  It is pinned against torch's own CPU
Philox engine (ATen PhiloxRNGEngine, an independent implementation that the
oracle does not share), compiled here from torch's installed headers, and by
distribution tests of the uniforms it yields.
"""
import os
import subprocess

import numpy as np
import pytest
import scipy.stats
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def torch_philox(tmp_path_factory):
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    exe = str(tmp_path_factory.mktemp("philox") / "torch_philox")
    subprocess.run(["g++", "-O1", "-std=c++17", "-I" + inc, "-o", exe,
                    os.path.join(HERE, "helpers", "torch_philox.cpp")], check=True)

    def run(queries):
        text = "".join(f"{s} {sub} {off} {n}\n" for s, sub, off, n in queries)
        out = subprocess.run([exe], input=text, capture_output=True, text=True, check=True).stdout
        return [list(map(int, line.split())) for line in out.strip().splitlines()]

    return run


def _cases(n, rng):
    seeds = rng.integers(0, 2**64, n, dtype=np.uint64)
    seeds[:4] = [0, 1, 0xFFFFFFFF, 0x123456789ABCDEF0]
    rows = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
    rows[:4] = [0, 1, 255, 0xFFFFFFFF]
    steps = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
    steps[:4] = [0, 11, 7, 0xFFFFFFFF]
    streams = rng.integers(0, 4, n).astype(np.uint32)
    vs = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
    vs[:8] = [0, 1, 2, 3, 4, 262143, 1023, 0xFFFFFFFF]
    return seeds, streams, steps, rows, vs


def test_philox_blocks_match_torch_engine(oracle_mod, torch_philox):
    """Full 128-bit blocks: oracle counter (c0,c1,c2,c3), key (k0,k1) equals
    torch's engine(seed=k0|k1<<32, subsequence=c2|c3<<32, offset=c0|c1<<32)."""
    rng = np.random.default_rng(1)
    n = 300
    ctrs = rng.integers(0, 2**32, (n, 4), dtype=np.uint64).astype(np.uint32)
    keys = rng.integers(0, 2**32, (n, 2), dtype=np.uint64).astype(np.uint32)
    ctrs[0] = 0
    keys[0] = 0
    ctrs[1] = 0xFFFFFFFF
    keys[1] = 0xFFFFFFFF
    got = oracle_mod.philox4x32_10(ctrs, keys)
    q = []
    for c, k in zip(ctrs.astype(np.uint64), keys.astype(np.uint64)):
        q.append((int(k[0] | (k[1] << 32)), int(c[2] | (c[3] << 32)), int(c[0] | (c[1] << 32)), 4))
    want = np.array(torch_philox(q), dtype=np.uint64).astype(np.uint32)
    np.testing.assert_array_equal(got, want)


def test_word_layout_matches_torch_engine(oracle_mod, torch_philox):
    """Word for (seed, stream, step, row, v): counter (v>>2, row, step,
    stream), output word v & 3."""
    rng = np.random.default_rng(2)
    seeds, streams, steps, rows, vs = _cases(200, rng)
    got = [int(oracle_mod.words(int(s), int(st), int(sp), [r], [v])[0])
           for s, st, sp, r, v in zip(seeds, streams, steps, rows, vs)]
    q = [(int(s), (int(st) << 32) | int(sp), (int(r) << 32) | (int(v) >> 2), (int(v) & 3) + 1)
         for s, st, sp, r, v in zip(seeds, streams, steps, rows, vs)]
    want = [ws[-1] for ws in torch_philox(q)]
    assert got == want


def test_uniforms_are_uniform(oracle_mod):
    """U = (2 (x >> 9) + 1) 2^-24 over consecutive vocab indices: KS test
    against U(0,1), and bucket counts of the top bits (chi-square)."""
    n = 200_000
    w = oracle_mod.words(0, 0, 3, np.full(n, 17, np.uint32), np.arange(n, dtype=np.uint32))
    u = (2.0 * (w >> 9).astype(np.float64) + 1.0) * 2.0**-24
    assert u.min() > 0.0 and u.max() < 1.0
    assert scipy.stats.kstest(u, "uniform").pvalue > 1e-3
    counts = np.bincount(w >> 24, minlength=256)
    assert scipy.stats.chisquare(counts).pvalue > 1e-3
    # the oracle's scalar mapping agrees on extreme words
    assert oracle_mod.uniform(0) == 2.0**-24
    assert oracle_mod.uniform(0xFFFFFFFF) == 1.0 - 2.0**-24


def test_streams_and_steps_are_decorrelated(oracle_mod):
    n = 100_000
    rows = np.arange(n, dtype=np.uint32)
    zeros = np.zeros(n, np.uint32)
    a = oracle_mod.words(0, 1, 0, rows, zeros).astype(np.float64)
    b = oracle_mod.words(0, 2, 0, rows, zeros).astype(np.float64)
    c = oracle_mod.words(0, 1, 1, rows, zeros).astype(np.float64)
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.02
    assert abs(np.corrcoef(a, c)[0, 1]) < 0.02
