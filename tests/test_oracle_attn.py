"""Pins for the oracle's canvas attention (float64).

Definition ("DiffusionGemma Technical Report", paperfeed review, "The
mechanism"): canvas queries attend bidirectionally to the whole canvas and
to the causally encoded cache; read here as one unmasked softmax over
[prefix_b || canvas_b] with GQA head h -> kv head h // (Hq / Hkv).

Pinned against: torch's float64 scaled_dot_product_attention (enable_gqa),
a pure-Python brute force on tiny inputs, closed forms, and the invariants
the method implies (canvas permutation equivariance, prefix permutation
invariance, zero-length prefix = self-attention, GQA = repeated-head MHA).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F


def _rand(shape, gen, dtype=torch.float32, gain=1.0):
    return (torch.randn(shape, generator=gen, dtype=torch.float32) * gain).to(dtype)


def _problem(B, C, Hq, Hkv, D, lens, seed=0, dtype=torch.float32, gain=1.0):
    g = torch.Generator().manual_seed(seed)
    q = _rand((B, C, Hq, D), g, dtype, gain)
    kc = _rand((B, C, Hkv, D), g, dtype)
    vc = _rand((B, C, Hkv, D), g, dtype)
    n = int(sum(lens))
    kp = _rand((n, Hkv, D), g, dtype)
    vp = _rand((n, Hkv, D), g, dtype)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return q, kc, vc, kp, vp, cu


def _sdpa(q, kc, vc, kp, vp, cu, scale):
    """Library reference: float64 SDPA per batch row on the concatenation."""
    B, C, Hq, D = q.shape
    outs, lses = [], []
    for b in range(B):
        k = torch.cat([kp[cu[b]:cu[b + 1]], kc[b]], 0).double()  # [L+C, Hkv, D]
        v = torch.cat([vp[cu[b]:cu[b + 1]], vc[b]], 0).double()
        qb = q[b].double().transpose(0, 1)                          # [Hq, C, D]
        o = F.scaled_dot_product_attention(qb, k.transpose(0, 1), v.transpose(0, 1),
                                           scale=scale, enable_gqa=True)
        outs.append(o.transpose(0, 1))
        group = Hq // k.shape[1]
        kk = k.transpose(0, 1).repeat_interleave(group, 0)
        s = scale * qb @ kk.transpose(1, 2)
        lses.append(torch.logsumexp(s, -1))
    return torch.stack(outs).numpy(), torch.stack(lses).numpy()


@pytest.mark.parametrize("B,C,Hq,Hkv,D,lens,dtype", [
    (1, 256, 2, 1, 64, (128,), torch.float32),       # the tiny workload's geometry
    (3, 24, 4, 2, 16, (0, 37, 130), torch.bfloat16),  # ragged, zero-length prefix
    (2, 40, 8, 2, 32, (5, 64), torch.float32),        # GQA 4:1
])
def test_matches_float64_sdpa(oracle_mod, B, C, Hq, Hkv, D, lens, dtype):
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=B * 7 + D, dtype=dtype)
    scale = 1.0 / math.sqrt(D)
    out, lse = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, scale)
    ref, ref_lse = _sdpa(q, kc, vc, kp, vp, cu, scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_brute_force_tiny(oracle_mod):
    """Pure-Python loops, one (b, i, h) at a time, C, L <= 8."""
    B, C, Hq, Hkv, D, lens = 2, 5, 2, 1, 4, (3, 8)
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=3)
    scale = 0.37
    out, _ = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, scale)
    qn, kcn, vcn, kpn, vpn = (t.numpy().tolist() for t in (q, kc, vc, kp, vp))
    for b in range(B):
        keys = [kpn[j][0] for j in range(cu[b], cu[b + 1])] + [kcn[b][j][0] for j in range(C)]
        vals = [vpn[j][0] for j in range(cu[b], cu[b + 1])] + [vcn[b][j][0] for j in range(C)]
        for i in range(C):
            for h in range(Hq):
                s = [scale * sum(a * c for a, c in zip(qn[b][i][h], k)) for k in keys]
                w = [math.exp(x) for x in s]
                tot = sum(w)
                o = [sum(w[j] * vals[j][d] for j in range(len(vals))) / tot for d in range(D)]
                np.testing.assert_allclose(out[b, i, h], o, rtol=1e-12, atol=1e-13)


def test_closed_forms(oracle_mod):
    B, C, Hq, Hkv, D, lens = 2, 16, 4, 2, 8, (10, 0)
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=5)
    # q = 0: uniform weights -> mean of all values of the kv head
    out, lse = oracle_mod.canvas_attn(torch.zeros_like(q), kc, vc, kp, vp, cu, 0.5)
    for b in range(B):
        v = torch.cat([vp[cu[b]:cu[b + 1]], vc[b]], 0).double().numpy()
        for h in range(Hq):
            np.testing.assert_allclose(out[b, :, h], np.broadcast_to(v[:, h // 2].mean(0), (C, D)),
                                       atol=1e-14)
            np.testing.assert_allclose(lse[b, h], math.log(v.shape[0]), atol=1e-14)
    # identical keys: weights uniform whatever q is
    kc1 = kc[:, :1].expand_as(kc).contiguous()
    kp1 = kc[0, 0].expand_as(kp).contiguous()
    out, _ = oracle_mod.canvas_attn(q, kc1, vc, kp1, vp, cu, 0.5)
    b = 0
    v = torch.cat([vp[cu[b]:cu[b + 1]], vc[b]], 0).double().numpy()
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(v[:, 0].mean(0), (C, D)), atol=1e-13)
    # a single key: the output is its value
    q1, kc1, vc1, kp0, vp0, cu0 = _problem(1, 1, 2, 1, 8, (0,), seed=9)
    out, _ = oracle_mod.canvas_attn(q1, kc1, vc1, kp0, vp0, cu0, 1.0)
    np.testing.assert_allclose(out[0, 0, 0], vc1[0, 0, 0].double().numpy(), atol=0)
    np.testing.assert_allclose(out[0, 0, 1], vc1[0, 0, 0].double().numpy(), atol=0)


def test_canvas_permutation_equivariance(oracle_mod):
    """No mask inside the canvas: permuting canvas rows of Q/Kc/Vc jointly
    permutes the output rows."""
    B, C, Hq, Hkv, D, lens = 2, 32, 4, 2, 16, (20, 7)
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=11, gain=3.0)
    perm = torch.randperm(C, generator=torch.Generator().manual_seed(0))
    out, lse = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.25)
    out_p, lse_p = oracle_mod.canvas_attn(q[:, perm].contiguous(), kc[:, perm].contiguous(),
                                          vc[:, perm].contiguous(), kp, vp, cu, 0.25)
    np.testing.assert_allclose(out_p, out[:, perm.numpy()], atol=1e-12)
    np.testing.assert_allclose(lse_p, lse[:, :, perm.numpy()], atol=1e-12)


def test_prefix_permutation_invariance(oracle_mod):
    B, C, Hq, Hkv, D, lens = 1, 16, 2, 1, 16, (50,)
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=12, gain=2.0)
    perm = torch.randperm(50, generator=torch.Generator().manual_seed(1))
    out, _ = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.25)
    out_p, _ = oracle_mod.canvas_attn(q, kc, vc, kp[perm].contiguous(), vp[perm].contiguous(),
                                      cu, 0.25)
    np.testing.assert_allclose(out_p, out, atol=1e-12)


def test_zero_prefix_is_self_attention(oracle_mod):
    B, C, Hq, Hkv, D = 2, 48, 4, 4, 16
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, (0, 0), seed=13)
    out, _ = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.25)
    for b in range(B):
        ref = F.scaled_dot_product_attention(q[b].double().transpose(0, 1),
                                             kc[b].double().transpose(0, 1),
                                             vc[b].double().transpose(0, 1), scale=0.25)
        np.testing.assert_allclose(out[b], ref.transpose(0, 1).numpy(), atol=1e-12)


def test_gqa_equals_repeated_heads(oracle_mod):
    B, C, Hq, Hkv, D, lens = 1, 20, 8, 2, 16, (33,)
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=14)
    out, _ = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.25)
    rep = Hq // Hkv
    out2, _ = oracle_mod.canvas_attn(q, kc.repeat_interleave(rep, 2), vc.repeat_interleave(rep, 2),
                                     kp.repeat_interleave(rep, 1), vp.repeat_interleave(rep, 1),
                                     cu, 0.25)
    np.testing.assert_array_equal(out, out2)


def test_position_subset_matches_full(oracle_mod):
    B, C, Hq, Hkv, D, lens = 2, 32, 4, 2, 16, (9, 40)
    q, kc, vc, kp, vp, cu = _problem(B, C, Hq, Hkv, D, lens, seed=15)
    out, lse = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.25)
    pos = [0, 7, 31]
    out_s, lse_s = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.25, positions=pos)
    np.testing.assert_array_equal(out_s[:, pos], out[:, pos])
    np.testing.assert_array_equal(lse_s[:, :, pos], lse[:, :, pos])
    assert np.isnan(out_s[:, 1]).all()


# ------------------------------------------------------------ 8-bit inputs
# E4M3 bytes (OCP "8-bit Floating Point Specification (OFP8)", E4M3 encoding:
# bias 7, three mantissa bits, subnormals m * 2^-9, S.1111.111 = NaN, no
# infinities) with one scale factor per tensor.

@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x3C, 1.5), (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0),
    (0xB8, -1.0), (0xFE, -448.0), (0x81, -(2.0 ** -9)),
])
def test_e4m3_closed_forms(oracle_mod, code, value):
    assert oracle_mod.e4m3_value(code) == value


def test_e4m3_nan_codes_and_negative_zero(oracle_mod):
    assert math.isnan(oracle_mod.e4m3_value(0x7F)) and math.isnan(oracle_mod.e4m3_value(0xFF))
    z = oracle_mod.e4m3_value(0x80)
    assert z == 0.0 and math.copysign(1.0, z) < 0


def test_e4m3_all_codes_match_torch(oracle_mod):
    """Every code against torch's float8_e4m3fn decoding (a library routine)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def _e4m3_problem(B, C, Hq, Hkv, D, lens, seed, gains=(40.0, 50.0, 30.0)):
    g = torch.Generator().manual_seed(seed)

    def r(*shape, gain):
        return (torch.randn(shape, generator=g) * gain).clamp(-448, 448).to(torch.float8_e4m3fn)

    n = int(sum(lens))
    q = r(B, C, Hq, D, gain=gains[0])
    kc, vc = r(B, C, Hkv, D, gain=gains[1]), r(B, C, Hkv, D, gain=gains[2])
    kp, vp = r(n, Hkv, D, gain=gains[1]), r(n, Hkv, D, gain=gains[2])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return q, kc, vc, kp, vp, cu


@pytest.mark.parametrize("B,C,Hq,Hkv,D,lens", [(2, 24, 4, 2, 32, (0, 45)),
                                               (1, 40, 8, 2, 16, (70,))])
def test_e4m3_scaled_matches_float64_sdpa(oracle_mod, B, C, Hq, Hkv, D, lens):
    """E4M3 inputs with distinct per-tensor factors against float64 SDPA on
    the decoded, scaled values (decoded by torch)."""
    q, kc, vc, kp, vp, cu = _e4m3_problem(B, C, Hq, Hkv, D, lens, seed=B + D)
    sq, sk, sv = 2.0 ** -5, 0.75 * 2.0 ** -6, 3.0 * 2.0 ** -7
    scale = 1.0 / math.sqrt(D)
    out, lse = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, scale, qkv_scale=(sq, sk, sv))
    dec = [t.to(torch.float64) * f for t, f in ((q, sq), (kc, sk), (vc, sv), (kp, sk), (vp, sv))]
    ref, ref_lse = _sdpa(*dec, cu, scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_e4m3_power_of_two_factors_equal_float32_path(oracle_mod):
    """Power-of-two factors scale exactly: the E4M3 path must equal the
    float32 path on the scaled values bit for bit."""
    q, kc, vc, kp, vp, cu = _e4m3_problem(2, 16, 4, 1, 8, (9, 20), seed=11)
    f = (2.0 ** -4, 2.0 ** -7, 2.0 ** -3)
    out, lse = oracle_mod.canvas_attn(q, kc, vc, kp, vp, cu, 0.3, qkv_scale=f)
    ts = [t.to(torch.float32) * s for t, s in ((q, f[0]), (kc, f[1]), (vc, f[2]), (kp, f[1]),
                                               (vp, f[2]))]
    out32, lse32 = oracle_mod.canvas_attn(*ts, cu, 0.3)
    np.testing.assert_array_equal(out, out32)
    np.testing.assert_array_equal(lse, lse32)
