"""GPU parity of the self-conditioning MLP (dd_ffw) and of the chained
dd_self_condition (soft embedding, then the MLP) against the float64
oracle ("DiffusionGemma Technical Report", paperfeed review, "The
mechanism", self-conditioning paragraph).

Tolerance (derived).  The kernels accumulate in fp32 and round twice to
bf16 (8 significant bits, unit roundoff 2^-8): the hidden activations and
the output.  Element-wise that gives
    |z_gpu - z| <= 2^-8 (|h| |W2|)_k + 2^-8 |z_k|
(h the float64 hidden layer; fp32 accumulation and erff add terms near
2^-23 relative, covered by a 5% margin and 1e-6).  With independent
rounding errors the relative RMS error is about 2^-8 / sqrt(3) per
rounding, sqrt(2) * 2.3e-3 = 3.2e-3 for the two: gate 8e-3.  The chained
call adds the soft embedding's own bf16 roundings (its tests measure
2-4e-3 relative RMS on u): gate 1.2e-2.
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_ffw(z_gpu, u, w1, b1, w2, b2):
    h = oracle._gelu64(_f64(u) @ _f64(w1) + _f64(b1))
    z = oracle.ffw(u.cpu(), w1.cpu(), b1.cpu(), w2.cpu(), b2.cpu())
    got = _f64(z_gpu)
    bound = 1.05 * 2.0 ** -8 * (np.abs(h) @ np.abs(_f64(w2)) + np.abs(z)) + 1e-6
    err = np.abs(got - z)
    assert (err <= bound).all(), f"max err/bound {float((err / bound).max()):.3f}"
    rel = float(np.sqrt((err ** 2).mean() / (z ** 2).mean()))
    assert rel <= 8e-3, f"relative RMS error {rel:.3e}"
    return rel


@pytest.mark.parametrize("rows,d,hidden", [(256, 2048, workloads.FFW_HIDDEN), (200, 128, 48),
                                           (1, 64, 16), (2048, 2048, workloads.FFW_HIDDEN),
                                           (300, 320, 1904)])
def test_ffw_matches_oracle(rows, d, hidden):
    w = workloads.scaled(workloads.WORKLOADS["b1_L4096"], name=f"ffw_{rows}_{d}_{hidden}")
    w1, b1, w2, b2 = (t.to(DEV) for t in workloads.ffw_weights(w, d, hidden))
    u = workloads.ffw_input(w, rows, d).to(DEV)
    z = dd.ffw(u, w1, b1, w2, b2)
    torch.cuda.synchronize()
    rel = _check_ffw(z, u, w1, b1, w2, b2)
    print(f"ffw rows {rows} d {d} h {hidden}: rel RMS {rel:.2e}")


def test_self_condition_matches_oracle_and_its_pieces():
    w = workloads.scaled(workloads.WORKLOADS["b1_L4096"], vocab=32768, name="selfcond")
    lg = workloads.logits(w, 0, device=DEV)
    E = workloads.embedding(w, device=DEV)
    w1, b1, w2, b2 = (t.to(DEV) for t in workloads.ffw_weights(w))
    tau = 0.8
    u = torch.empty((w.rows, E.shape[1]), dtype=torch.bfloat16, device=DEV)
    z = dd.self_condition(lg, tau, E, w1, b1, w2, b2, u_out=u)
    torch.cuda.synchronize()
    # the same kernels one by one give the same bits
    assert torch.equal(u, dd.soft_embed(lg, tau, E))
    assert torch.equal(z, dd.ffw(u, w1, b1, w2, b2))
    ref = oracle.self_condition(lg.cpu(), tau, E.cpu(), w1.cpu(), b1.cpu(), w2.cpu(), b2.cpu())
    err = _f64(z) - ref
    rel = float(np.sqrt((err ** 2).mean() / (ref ** 2).mean()))
    print(f"self condition: rel RMS {rel:.2e}")
    assert rel <= 1.2e-2, f"relative RMS error {rel:.3e}"
    # without u_out the soft embedding goes to the workspace: same result
    assert torch.equal(dd.self_condition(lg, tau, E, w1, b1, w2, b2), z)


def test_ffw_rejects_bad_shapes():
    w = workloads.WORKLOADS["b1_L4096"]
    w1, b1, w2, b2 = (t.to(DEV) for t in workloads.ffw_weights(w, 64, 16))
    u = workloads.ffw_input(w, 4, 64).to(DEV)
    lib = dd.load()
    ws = dd.new_workspace(int(lib.dd_ffw_workspace(4, 64, 16)), DEV)
    out = torch.empty_like(u)
    args = lambda d, h: (dd._ptr(u), 4, d, h, dd._ptr(w1), dd._ptr(b1), dd._ptr(w2), dd._ptr(b2),
                         dd._ptr(out), dd._ptr(ws), ws.numel(), None)
    assert lib.dd_ffw(*args(64, 24)) == 2          # hidden not a multiple of 16
    assert lib.dd_ffw(*args(8, 16)) == 1           # d below 16
    assert lib.dd_ffw(*args(64, 16)) == 0
    torch.cuda.synchronize()
