"""Comparison rules between the CUDA path and the oracle.

Tolerances:
  attention, bf16 inputs : max |err| <= 2e-2 (acceptance bound) and relative
                           RMS error <= 1e-2 (an internal gate; with N(0,1)
                           inputs the outputs are ~0.02 in size, so the
                           absolute bound alone would be weak)
  attention, fp32 inputs : max |err| <= 1e-5
  attention, E4M3 inputs : the kernel rounds each softmax probability P to
                           E4M3 for the P.V product (relative error <= 2^-4
                           in E4M3's normal range; P >= 2^-6 * max P is
                           normal, smaller P err by <= 2^-10 absolute with
                           max P >= 2^6).  With independent rounding errors
                           the output's relative RMS error is about
                           2^-4 / sqrt(3) * E[1/m^2]^(1/2) ~ 0.026 (m the
                           mantissa in [1, 2)), at most 2^-4 / sqrt(3) =
                           0.036: gate 5e-2.  Max |err| <= max|V| (2^-4 +
                           n_keys 2^-16) + 2^-8 max|O| (the bf16 output)
                           bounds it rigorously.
  confidence             : relative error <= 1e-5
  entropy                : |err| <= 1e-5 * max(1, |H|)
  token ids              : bit-exact, except a sampled id at a position that
                           is NOT re-noised and whose two best Gumbel scores
                           (float64, oracle) differ by < 1e-5: such near-ties
                           are counted and reported, not failed.  Re-noise
                           decisions and replacement ids never depend on the
                           scores and are always bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

NEAR_TIE = 1e-5


def _np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().numpy()
    return np.asarray(x)


def check_sampler(got: dict, ref: dict, rows=None, conf_rtol=1e-5, ent_tol=1e-5) -> dict:
    """got: device tensors from the library; ref: oracle dict (rows = the
    local row indices the oracle computed, None = all)."""
    sel = slice(None) if rows is None else np.asarray(rows)
    tokens = _np(got["tokens"])[sel]
    renoised = _np(got["renoised"])[sel] if got.get("renoised") is not None else None
    pred = _np(got["pred"])[sel] if got.get("pred") is not None else None
    conf = _np(got["conf"])[sel].astype(np.float64)
    if renoised is not None:
        np.testing.assert_array_equal(renoised, ref["renoised"], err_msg="re-noise decisions")
    rn = ref["renoised"].astype(bool)
    # replacement ids: exact
    np.testing.assert_array_equal(tokens[rn], ref["tokens"][rn], err_msg="replacement ids")
    near = ref["gap"] < NEAR_TIE
    p = pred if pred is not None else np.where(rn, ref["pred"], tokens)
    mism = p != ref["pred"]
    bad = mism & ~near
    assert not bad.any(), (f"{int(bad.sum())} sampled ids differ away from near-ties; rows "
                           f"{np.nonzero(bad)[0][:10]} gaps {ref['gap'][bad][:10]}")
    keep_ok = ~rn & ~mism
    np.testing.assert_array_equal(tokens[~rn & ~near], ref["tokens"][~rn & ~near])
    same = ~mism
    rel = np.abs(conf[same] - ref["conf"][same]) / np.abs(ref["conf"][same])
    assert rel.size == 0 or rel.max() <= conf_rtol, f"conf rel err {rel.max():.3e}"
    if got.get("entropy") is not None:
        ent = _np(got["entropy"])[sel].astype(np.float64)
        err = np.abs(ent - ref["entropy"]) / np.maximum(1.0, np.abs(ref["entropy"]))
        assert err.max() <= ent_tol, f"entropy err {err.max():.3e}"
    return {"rows": int(tokens.size), "near_ties": int(near.sum()),
            "near_tie_mismatches": int(mism.sum()), "kept_exact": int(keep_ok.sum()),
            "conf_max_rel": float(rel.max()) if rel.size else 0.0}


FP8_REL_RMS = 5e-2


def fp8_max_abs(v_max: float, n_keys: int, o_max: float) -> float:
    """The E4M3 path's rigorous max |err| bound (see the module docstring)."""
    return v_max * (2.0 ** -4 + n_keys * 2.0 ** -16) + 2.0 ** -8 * o_max


def check_attn(got, ref, dtype, positions=None, max_abs=None, rel_rms=1e-2) -> dict:
    """got: [B,C,Hq,D] device tensor; ref: oracle float64 array."""
    g = _np(got.float())
    r = ref
    if positions is not None:
        g = g[:, positions]
        r = r[:, positions]
    err = np.abs(g.astype(np.float64) - r)
    mx = float(err.max())
    rrms = float(np.sqrt((err ** 2).mean() / max((r ** 2).mean(), 1e-30)))
    bound = max_abs if max_abs is not None else (2e-2 if dtype == torch.bfloat16 else 1e-5)
    assert mx <= bound, f"max abs err {mx:.3e} > {bound}"
    if dtype == torch.bfloat16:
        assert rrms <= rel_rms, f"relative RMS err {rrms:.3e} > {rel_rms}"
    return {"max_abs": mx, "rel_rms": rrms}
