"""GPU parity of dd_soft_embed (self-conditioning soft embedding,
softmax(logits / tau) E) against the float64 oracle.

Tolerances (derived from the arithmetic; bf16 keeps 8 significant bits, so
its unit roundoff is 2^-8): each probability is rounded to bf16 for the
tensor-core product (relative error <= 2^-8), accumulation is fp32 and the
output is rounded to bf16 (<= 2^-8 of |out|), so per element
|err| <= 2^-8 max|E| + 2^-7 max|out|.  With independent rounding errors the
relative RMS error is about 2^-8 / sqrt(3) * 0.72 ~ 1.6e-3 for each of the
two roundings, ~2.3e-3 together; when one probability dominates a row the
errors do not average and the relative error reaches 2 * 2^-8: gate 8e-3.  Sizes span ragged row blocks (< 256 rows,
> 256 rows), a vocabulary that is not a multiple of the 64-entry step, a
padded row stride, embedding widths below and above the 256-column tile,
and the full 256 x 262,144 workload on sampled rows and columns.
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _check(got, ref, E, rel_rms=8e-3):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    bound = 2.0 ** -8 * float(E.float().abs().max()) + 2.0 ** -7 * float(np.abs(ref).max())
    assert err.max() <= bound, f"max abs err {err.max():.3e} > {bound:.3e}"
    rr = float(np.sqrt((err ** 2).mean() / max((ref ** 2).mean(), 1e-30)))
    assert rr <= rel_rms, f"relative RMS err {rr:.3e}"
    return {"max_abs": float(err.max()), "rel_rms": rr}


def _inputs(R, V, d, seed, lscale=3.0, stride=None):
    g = torch.Generator().manual_seed(seed)
    st = V if stride is None else stride
    lg = (torch.randn((R, st), generator=g) * lscale).to(torch.bfloat16)
    E = torch.randn((V, d), generator=g).to(torch.bfloat16)
    return lg, E


@pytest.mark.parametrize("R,V,d,tau,stride", [
    (37, 1000, 128, 0.8, None),     # one partial row block, ragged vocabulary, d < 256
    (300, 5000, 320, 1.0, 5008),    # two row blocks, padded stride, ragged column tile
    (256, 4096, 512, 1.7, None),    # exact tiles
])
def test_soft_embed_small(R, V, d, tau, stride):
    lg, E = _inputs(R, V, d, seed=R + d, stride=stride)
    out = dd.soft_embed(lg.to(DEV), tau, E.to(DEV), vocab=V)
    torch.cuda.synchronize()
    ref = oracle.soft_embed(lg[:, :V].contiguous(), tau, E)
    print(R, V, d, _check(out, ref, E))


def test_soft_embed_dominant_logit_returns_the_row():
    R, V, d = 64, 3000, 256
    lg, E = _inputs(R, V, d, seed=5)
    idx = torch.randint(0, V, (R,), generator=torch.Generator().manual_seed(6))
    lg[torch.arange(R), idx] = 120.0
    out = dd.soft_embed(lg.to(DEV), 1.0, E.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.soft_embed(lg, 1.0, E)
    _check(out, ref, E)
    # the bf16 result is the selected row itself (probability 1 exactly)
    assert torch.equal(out.cpu(), E[idx])


def test_soft_embed_full_workload_sampled():
    w = workloads.WORKLOADS["b1_L4096"]
    lg = workloads.logits(w, 0, device=DEV)
    E = workloads.embedding(w, device=DEV)
    ws = dd.new_workspace(dd.soft_embed_workspace_bytes(w.rows, w.vocab, E.shape[1]))
    out = dd.soft_embed(lg, 1.0, E, workspace=ws)
    dd.query_device_error(ws)
    rows = np.array([0, 1, 77, 255])
    cols = np.unique(np.random.default_rng(0).integers(0, E.shape[1], 96))
    ref = oracle.soft_embed(lg.cpu()[rows], 1.0, E.cpu(), cols=cols)
    st = _check(out[rows][:, cols], ref, E)
    print("full", st)
