"""Writes the regression fixtures in this directory from the oracle.

    python tests/golden/make_golden.py

The pages ("DiffusionGemma Technical Report", paperfeed review) print no
worked example of the step's arithmetic, so no fixture here holds the pages'
own numbers.  These fixtures freeze what the float64 oracle computes on small
seeded inputs that reach every branch of the step: a ragged vocabulary tail,
an empty prefix, grouped heads, a spiked row, re-noised and kept positions.
The oracle itself is pinned elsewhere against independent references (torch's
Philox engine, float64 SDPA, closed forms, distribution tests).  A change to
the oracle's arithmetic therefore shows up as a failing regression test and a
diff of a committed file, and the CUDA library is checked against the same
stored values (tests/test_golden_gpu.py).

Only the oracle computes the stored outputs.  numpy's seeded generator makes
the inputs, which are stored beside the outputs, so a fixture does not depend
on the generator's stream staying the same.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402

PAGES = '"DiffusionGemma Technical Report" (paperfeed review)'


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _write(name: str, obj: dict) -> None:
    path = os.path.join(HERE, name)
    with open(path, "w") as f:
        json.dump(obj, f, indent=None, separators=(",", ":"))
        f.write("\n")
    print(f"wrote {path} ({os.path.getsize(path)} bytes)")


def philox() -> dict:
    rng = np.random.default_rng(101)
    ctr = rng.integers(0, 2**32, (6, 4), dtype=np.uint64).astype(np.uint32)
    key = rng.integers(0, 2**32, (6, 2), dtype=np.uint64).astype(np.uint32)
    ctr[0] = 0
    key[0] = 0
    ctr[1] = 0xFFFFFFFF
    key[1] = 0xFFFFFFFF
    blocks = oracle.philox4x32_10(ctr, key)
    seeds = [0, 1, 0x123456789ABCDEF0]
    streams = [0, 1, 2, 3]
    rows = np.array([0, 1, 255, 0xFFFFFFFF], np.uint32)
    vs = np.array([0, 3, 4, 262143], np.uint32)
    wl = []
    for s in seeds:
        for st in streams:
            w = oracle.words(s, st, 7, rows, vs)
            wl.append({"seed": s, "stream": st, "step": 7, "rows": rows.tolist(),
                       "v": vs.tolist(), "words": w.tolist(),
                       "uniform": [oracle.uniform(int(x)) for x in w]})
    return {
        "source": "Salmon et al., 'Parallel random numbers: as easy as 1, 2, 3' (SC'11), "
                  "Philox4x32-10; the counter layout (v >> 2, row, step, stream) and the "
                  f"uniform map are this library's reading of {PAGES}, 'The mechanism'",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "blocks": [{"counter": c.tolist(), "key": k.tolist(), "out": o.tolist()}
                   for c, k, o in zip(ctr, key, blocks)],
        "words": wl,
    }


def _g13(a) -> list:
    """float64 values to 13 significant digits (relative error < 5e-13)."""
    return [float(f"{v:.13g}") for v in np.asarray(a, np.float64).ravel()]


def attention() -> dict:
    rng = np.random.default_rng(202)
    B, C, Hq, Hkv, D = 2, 5, 2, 1, 128
    lens = [3, 0]
    n = sum(lens)

    def bf16(*shape, gain=1.0):
        return bf16_bits((rng.standard_normal(shape) * gain).astype(np.float32))

    q, kc, vc = bf16(B, C, Hq, D, gain=2.0), bf16(B, C, Hkv, D), bf16(B, C, Hkv, D)
    kp, vp = bf16(n, Hkv, D), bf16(n, Hkv, D)
    cu = np.array([0, 3, 3], np.int32)
    scale = 128 ** -0.5
    out, lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu, scale)
    return {
        "source": f"{PAGES}, 'The mechanism': bidirectional attention of every canvas "
                  "position over the block's prefix cache and the whole canvas",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "shape": {"B": B, "C": C, "Hq": Hq, "Hkv": Hkv, "D": D}, "prefix_lens": lens,
        "scale": scale, "dtype": "bf16",
        "q": q.ravel().tolist(), "kc": kc.ravel().tolist(), "vc": vc.ravel().tolist(),
        "kp": kp.ravel().tolist(), "vp": vp.ravel().tolist(), "cu_prefix": cu.tolist(),
        "out": _g13(out), "lse": _g13(lse),
    }


def sampler() -> dict:
    rng = np.random.default_rng(303)
    R, V = 6, 300
    x = (rng.standard_normal((R, V)) * 3.0).astype(np.float32)
    x[1, 17] += 12.0           # one dominant entry
    x[2, 299] += 12.0          # dominant entry in the ragged tail
    x[3] = 0.5                 # constant row: uniform distribution
    bits = bf16_bits(x)
    cases = []
    for tau, rate, seed, step in [(1.0, 0.0, 5, 0), (0.7, 0.5, 5, 3), (1.3, 1.0, 9, 11)]:
        r = oracle.sample_renoise(bits, tau, rate, seed, step)
        cases.append({"tau": tau, "rate": rate, "seed": seed, "step": step,
                      **{k: r[k].tolist() for k in ("tokens", "pred", "renoised")},
                      **{k: _g13(r[k]) for k in ("conf", "entropy", "gap")}})
    return {
        "source": f"{PAGES}, 'The mechanism': temperature-scaled logits, per-position "
                  "entropy, tokens that are not kept re-noised to uniform vocabulary ids",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "rows": R, "vocab": V, "dtype": "bf16", "logits_bf16": bits.ravel().tolist(),
        "cases": cases,
        "init_canvas": {"rows": 7, "vocab": 1000, "seed": 42, "row_offset": 3,
                        "canvas": oracle.init_canvas(7, 1000, 42, 3).tolist()},
    }


def policy() -> dict:
    rng = np.random.default_rng(404)
    B, C, V = 2, 16, 500
    ent = (rng.exponential(0.05, B * C)).astype(np.float32)
    ent[3] = 0.0
    ent[C + 5] = 2.0
    pred = rng.integers(0, V, B * C).astype(np.int32)
    acc = oracle.entropy_accept(ent, pred, C, 0.1, 8, 2, V)
    prev = pred.copy()
    prev[C + 1] += 1           # canvas 1 changed a prediction
    small = np.full(B * C, 1e-3, np.float32)
    done = oracle.stop_check(small, pred, prev, C, 0.005)
    return {
        "source": f"{PAGES}, 'The mechanism', sampler paragraph: entropy-bounded "
                  "acceptance under a budget, and the early halt when entropies and "
                  "predictions have settled",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "batch": B, "canvas": C, "vocab": V, "budget": 0.1, "seed": 8, "step": 2,
        "entropy": ent.tolist(), "pred": pred.tolist(),
        "tokens": acc["tokens"].tolist(), "accepted": acc["accepted"].tolist(),
        "n_accepted": acc["n_accepted"].tolist(), "sum_accepted": _g13(acc["sum_accepted"]),
        "stop": {"entropy": small.tolist(), "pred_prev": prev.tolist(), "threshold": 0.005,
                 "done": done.tolist()},
    }


def soft_embedding() -> dict:
    rng = np.random.default_rng(505)
    R, V, d = 3, 37, 64
    lg = bf16_bits((rng.standard_normal((R, V)) * 2.0).astype(np.float32))
    E = bf16_bits(rng.standard_normal((V, d)).astype(np.float32))
    tau = 0.8
    out = oracle.soft_embed(lg, tau, E)
    return {
        "source": f"{PAGES}, 'The mechanism', self-conditioning paragraph: the step's "
                  "predicted distribution pushed through the embedding matrix",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "rows": R, "vocab": V, "d": d, "tau": tau, "dtype": "bf16",
        "logits_bf16": lg.ravel().tolist(), "emb_bf16": E.ravel().tolist(),
        "out": _g13(out),
    }


def main() -> None:
    oracle.build()
    _write("philox.json", philox())
    _write("canvas_attn.json", attention())
    _write("sampler.json", sampler())
    _write("policy.json", policy())
    _write("soft_embed.json", soft_embedding())


if __name__ == "__main__":
    main()
