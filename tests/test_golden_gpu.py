"""The CUDA library on the inputs of the committed fixtures (tests/golden/),
against the oracle values stored there, with the same gates as the parity
tests: integer work exact (sampled ids away from near-ties), floating point
within the tolerances tests/parity.py and tests/test_soft_embed_gpu.py
derive."""
import json
import os

import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
from parity import check_attn, check_sampler

pytestmark = pytest.mark.gpu

DEV = "cuda"
HERE = os.path.dirname(os.path.abspath(__file__))


def _load(name):
    with open(os.path.join(HERE, "golden", name)) as f:
        return json.load(f)


def _bf16(xs, shape):
    a = np.asarray(xs, np.uint16).reshape(shape).view(np.int16)
    return torch.from_numpy(a.copy()).view(torch.bfloat16).to(DEV)


def test_canvas_attn_golden():
    d = _load("canvas_attn.json")
    s = d["shape"]
    B, C, Hq, Hkv, D = s["B"], s["C"], s["Hq"], s["Hkv"], s["D"]
    n = sum(d["prefix_lens"])
    cu = np.array(d["cu_prefix"], np.int32)
    out, lse = dd.canvas_attn(_bf16(d["q"], (B, C, Hq, D)), _bf16(d["kc"], (B, C, Hkv, D)),
                              _bf16(d["vc"], (B, C, Hkv, D)), _bf16(d["kp"], (n, Hkv, D)),
                              _bf16(d["vp"], (n, Hkv, D)), torch.from_numpy(cu).to(DEV), cu,
                              scale=d["scale"], want_lse=True)
    torch.cuda.synchronize()
    ref = np.asarray(d["out"]).reshape(B, C, Hq, D)
    print(check_attn(out, ref, torch.bfloat16))
    np.testing.assert_allclose(lse.cpu().numpy().ravel(), d["lse"], atol=1e-3)


def test_sampler_golden():
    d = _load("sampler.json")
    lg = _bf16(d["logits_bf16"], (d["rows"], d["vocab"]))
    for c in d["cases"]:
        got = dd.sample_renoise(lg, c["tau"], c["rate"], c["seed"], c["step"])
        torch.cuda.synchronize()
        ref = {k: np.asarray(c[k]) for k in ("tokens", "pred", "conf", "entropy", "renoised",
                                             "gap")}
        st = check_sampler(got, ref)
        assert st["near_tie_mismatches"] == 0, st
    ic = d["init_canvas"]
    got = dd.init_canvas(ic["rows"], ic["vocab"], ic["seed"], ic["row_offset"])
    assert got.cpu().tolist() == ic["canvas"]


def test_policy_golden():
    d = _load("policy.json")
    h = torch.tensor(d["entropy"], dtype=torch.float32, device=DEV)
    pred = torch.tensor(d["pred"], dtype=torch.int32, device=DEV)
    acc = dd.entropy_accept(h, pred, d["canvas"], d["budget"], d["seed"], d["step"], d["vocab"])
    torch.cuda.synchronize()
    assert acc["accepted"].cpu().tolist() == d["accepted"]
    assert acc["tokens"].cpu().tolist() == d["tokens"]
    st = d["stop"]
    B = d["batch"]
    done = torch.zeros(B, dtype=torch.uint8, device=DEV)
    halt = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    dd.stop_check(torch.tensor(st["entropy"], dtype=torch.float32, device=DEV), pred,
                  torch.tensor(st["pred_prev"], dtype=torch.int32, device=DEV), d["canvas"],
                  st["threshold"], 3, done, halt)
    assert done.cpu().tolist() == st["done"]
    assert halt.cpu().tolist() == [3 if x else -1 for x in st["done"]]


def test_soft_embed_golden():
    d = _load("soft_embed.json")
    R, V, dim = d["rows"], d["vocab"], d["d"]
    lg = torch.zeros((R, 40), dtype=torch.bfloat16, device=DEV)   # row stride 40 (16-byte rows)
    lg[:, :V] = _bf16(d["logits_bf16"], (R, V))
    E = _bf16(d["emb_bf16"], (V, dim))
    out = dd.soft_embed(lg, d["tau"], E, vocab=V)
    torch.cuda.synchronize()
    ref = np.asarray(d["out"]).reshape(R, dim)
    err = np.abs(out.float().cpu().numpy().astype(np.float64) - ref)
    bound = 2.0 ** -8 * float(E.float().abs().max()) + 2.0 ** -7 * float(np.abs(ref).max())
    assert err.max() <= bound
    rr = float(np.sqrt((err ** 2).mean() / (ref ** 2).mean()))
    assert rr <= 8e-3, rr
