"""GPU parity of dd_canvas_attn_fp8 (E4M3 inputs, per-tensor factors) against
the float64 oracle on the decoded, scaled inputs.

The 8-bit path runs the same tcgen05 kernel as bf16 with kind::f8f6f4 MMAs:
Q.K^T on E4M3 operands, P rounded to E4M3 for P.V.  Sizes span several
128-key and 128-row tiles with ragged tails, zero-length prefixes, canvases
that are not a multiple of 128, the head groupings the kernel takes, a
sharp softmax (Q x 4: few keys dominate, the running-max rescale runs), and
the full workloads in their real launch configuration on sampled positions.
Tolerances: tests/parity.py (derived from the E4M3 rounding of P).
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads
from parity import FP8_REL_RMS, check_attn, fp8_max_abs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _problem(B, C, Hq, Hkv, D, lens, seed=0, q_gain=1.0):
    g = torch.Generator().manual_seed(seed)

    def r(*shape, gain=1.0):
        return torch.randn(shape, generator=g) * gain

    n = int(sum(lens))
    (q,), fq = workloads.to_e4m3([r(B, C, Hq, D, gain=q_gain)])
    (kc, kp), fk = workloads.to_e4m3([r(B, C, Hkv, D), r(n, Hkv, D)])
    (vc, vp), fv = workloads.to_e4m3([r(B, C, Hkv, D), r(n, Hkv, D)])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    return q, kc, vc, kp, vp, cu, (fq, fk, fv)


def _check(out, ref, vc, vp, fv, n_keys, positions=None):
    v_max = fv * max(float(vc.float().abs().max()),
                     float(vp.float().abs().max()) if vp.numel() else 0.0)
    bound = fp8_max_abs(v_max, n_keys, float(np.nanmax(np.abs(ref))))
    return check_attn(out, ref, torch.bfloat16, positions=positions, max_abs=bound,
                      rel_rms=FP8_REL_RMS)


def _run(q, kc, vc, kp, vp, cu, f, scale=None):
    desc = dd.attn_desc(q, kc, scale)
    ws = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, cu))
    out, lse = dd.canvas_attn_fp8(q.to(DEV), kc.to(DEV), vc.to(DEV), kp.to(DEV), vp.to(DEV),
                                  cu.to(DEV), f, cu, scale=scale, want_lse=True, workspace=ws)
    dd.query_device_error(ws)  # synchronises; raises on a latched device error
    assert out.dtype == torch.bfloat16
    return out, lse


@pytest.mark.parametrize("lens,q_gain", [((0, 100, 300), 1.0), ((129, 1, 640), 4.0),
                                         ((4096,), 1.0), ((1000,), 4.0)])
def test_fp8_ragged(lens, q_gain):
    B = len(lens)
    q, kc, vc, kp, vp, cu, f = _problem(B, 256, 16, 8, 128, lens, seed=len(lens) + 10,
                                        q_gain=q_gain)
    out, lse = _run(q, kc, vc, kp, vp, cu, f)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5, qkv_scale=f)
    st = _check(out, ref, vc, vp, f[2], max(lens) + 256)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=1e-3)
    print(lens, q_gain, st)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (16, 2), (32, 4)])
def test_fp8_head_groupings(Hq, Hkv):
    q, kc, vc, kp, vp, cu, f = _problem(2, 256, Hq, Hkv, 128, (200, 77), seed=Hq + Hkv + 20)
    out, _ = _run(q, kc, vc, kp, vp, cu, f)
    ref, _ = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5, qkv_scale=f)
    _check(out, ref, vc, vp, f[2], 456)


@pytest.mark.parametrize("C", [200, 64, 1])
def test_fp8_ragged_canvas(C):
    q, kc, vc, kp, vp, cu, f = _problem(2, C, 16, 8, 128, (150, 0), seed=C + 30)
    out, _ = _run(q, kc, vc, kp, vp, cu, f)
    ref, _ = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5, qkv_scale=f)
    _check(out, ref, vc, vp, f[2], 150 + C)


def test_fp8_factors_enter_as_stated():
    """Halving f_v halves O exactly (a power-of-two factor of the bf16
    result); doubling f_q and halving f_k leaves O unchanged."""
    q, kc, vc, kp, vp, cu, f = _problem(1, 256, 16, 8, 128, (300,), seed=41, q_gain=2.0)
    out, lse = _run(q, kc, vc, kp, vp, cu, f)
    out_v, _ = _run(q, kc, vc, kp, vp, cu, (f[0], f[1], f[2] / 2))
    assert torch.equal(out_v.float() * 2, out.float())
    out_qk, lse_qk = _run(q, kc, vc, kp, vp, cu, (f[0] * 2, f[1] / 2, f[2]))
    assert torch.equal(out_qk, out) and torch.equal(lse_qk, lse)


def _positions(C, n=12, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, 1, C - 1], rng.integers(0, C, n)])).astype(np.int32)


@pytest.mark.parametrize("name", ["b1_L4096", "long_L65536", "ragged_b8"])
def test_fp8_full_workloads_sampled(name):
    w = workloads.WORKLOADS[name]
    q, kc, vc, kp, vp, cu, f = workloads.e4m3_attn_inputs(w, 0, device=DEV)
    out, lse = dd.canvas_attn_fp8(q, kc, vc, kp, vp, cu.to(DEV), f, cu, scale=w.scale,
                                  want_lse=True)
    torch.cuda.synchronize()
    pos = _positions(w.canvas, 6 if name == "long_L65536" else 12)
    ref, ref_lse = oracle.canvas_attn(q.cpu(), kc.cpu(), vc.cpu(), kp.cpu(), vp.cpu(),
                                      cu.numpy(), w.scale, positions=pos, qkv_scale=f)
    st = _check(out, ref, vc, vp, f[2], max(w.prefix_lens) + w.canvas, positions=pos)
    np.testing.assert_allclose(lse.cpu().numpy()[:, :, pos], ref_lse[:, :, pos], atol=1e-3)
    print(name, st)
