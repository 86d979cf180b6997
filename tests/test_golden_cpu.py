"""The oracle reproduces the committed fixtures in tests/golden/.

The fixtures were written by tests/golden/make_golden.py, which calls the
oracle only (the pages print no worked example).  Integer outputs must match
exactly; float64 outputs to the 13 significant digits stored.  A failure
here means the oracle's arithmetic changed: regenerate the fixtures only
with a commit that names the passage, or the reading of it, behind the
change.
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
RTOL = 1e-12


def _load(name):
    with open(os.path.join(HERE, "golden", name)) as f:
        return json.load(f)


def _u16(xs, shape):
    return np.asarray(xs, np.uint16).reshape(shape)


@pytest.mark.parametrize("name", ["philox.json", "canvas_attn.json", "sampler.json",
                                  "policy.json", "soft_embed.json"])
def test_fixture_states_its_source(name):
    d = _load(name)
    assert "DiffusionGemma" in d["source"] or "Salmon" in d["source"]
    assert d["written_by"].startswith("tests/golden/make_golden.py")


def test_philox_fixture(oracle_mod):
    d = _load("philox.json")
    for b in d["blocks"]:
        got = oracle_mod.philox4x32_10(np.array([b["counter"]], np.uint32),
                                       np.array([b["key"]], np.uint32))
        assert got[0].tolist() == b["out"]
    for w in d["words"]:
        got = oracle_mod.words(w["seed"], w["stream"], w["step"], np.array(w["rows"], np.uint32),
                               np.array(w["v"], np.uint32))
        assert got.tolist() == w["words"]
        assert [oracle_mod.uniform(x) for x in got] == w["uniform"]


def test_canvas_attn_fixture(oracle_mod):
    d = _load("canvas_attn.json")
    s = d["shape"]
    B, C, Hq, Hkv, D = s["B"], s["C"], s["Hq"], s["Hkv"], s["D"]
    n = sum(d["prefix_lens"])
    out, lse = oracle_mod.canvas_attn(
        _u16(d["q"], (B, C, Hq, D)), _u16(d["kc"], (B, C, Hkv, D)), _u16(d["vc"], (B, C, Hkv, D)),
        _u16(d["kp"], (n, Hkv, D)), _u16(d["vp"], (n, Hkv, D)), np.array(d["cu_prefix"]),
        d["scale"])
    np.testing.assert_allclose(out.ravel(), d["out"], rtol=RTOL, atol=1e-300)
    np.testing.assert_allclose(lse.ravel(), d["lse"], rtol=RTOL)


def test_sampler_fixture(oracle_mod):
    d = _load("sampler.json")
    lg = _u16(d["logits_bf16"], (d["rows"], d["vocab"]))
    for c in d["cases"]:
        r = oracle_mod.sample_renoise(lg, c["tau"], c["rate"], c["seed"], c["step"])
        for k in ("tokens", "pred", "renoised"):
            assert r[k].tolist() == c[k], k
        for k in ("conf", "entropy", "gap"):
            np.testing.assert_allclose(r[k], c[k], rtol=RTOL, err_msg=k)
    ic = d["init_canvas"]
    got = oracle_mod.init_canvas(ic["rows"], ic["vocab"], ic["seed"], ic["row_offset"])
    assert got.tolist() == ic["canvas"]


def test_policy_fixture(oracle_mod):
    d = _load("policy.json")
    acc = oracle_mod.entropy_accept(np.array(d["entropy"], np.float32), np.array(d["pred"]),
                                    d["canvas"], d["budget"], d["seed"], d["step"], d["vocab"])
    for k in ("tokens", "accepted", "n_accepted"):
        assert acc[k].tolist() == d[k], k
    np.testing.assert_allclose(acc["sum_accepted"], d["sum_accepted"], rtol=RTOL)
    st = d["stop"]
    done = oracle_mod.stop_check(np.array(st["entropy"], np.float32), np.array(d["pred"]),
                                 np.array(st["pred_prev"]), d["canvas"], st["threshold"])
    assert done.tolist() == st["done"]


def test_soft_embed_fixture(oracle_mod):
    d = _load("soft_embed.json")
    out = oracle_mod.soft_embed(_u16(d["logits_bf16"], (d["rows"], d["vocab"])), d["tau"],
                                _u16(d["emb_bf16"], (d["vocab"], d["d"])))
    np.testing.assert_allclose(out.ravel(), d["out"], rtol=RTOL, atol=1e-15)


def test_fixtures_cover_the_branches():
    """The sampler fixture holds kept and re-noised rows, the attention
    fixture an empty prefix, the policy fixture accepted and rejected
    positions and both halt outcomes."""
    s = _load("sampler.json")
    rn = np.concatenate([c["renoised"] for c in s["cases"]])
    assert rn.any() and not rn.all()
    assert s["vocab"] % 256 != 0
    a = _load("canvas_attn.json")
    assert 0 in a["prefix_lens"] and a["shape"]["Hq"] > a["shape"]["Hkv"]
    p = _load("policy.json")
    assert 0 < sum(p["accepted"]) < len(p["accepted"])
    assert sorted(set(p["stop"]["done"])) == [0, 1]
