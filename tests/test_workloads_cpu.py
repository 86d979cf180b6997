"""The seeded input generators: same seeds give the same bits, the shapes and
distributions stated in the workloads module, and the 8-bit inputs' scale
factors as stated (powers of two, one K and one V factor over the prefix and
every step of a block)."""
import dataclasses
import math

import numpy as np
import torch

import workloads

SMALL = workloads.scaled(workloads.WORKLOADS["block12_L8192"], prefix_lens=(300,), vocab=2000,
                         steps=3, rates=(0.9, 0.4, 0.0), temperatures=(1.0, 0.8, 0.7),
                         name="block3_small")


def _is_pow2(f):
    return f > 0 and math.frexp(f)[0] == 0.5


def test_same_seed_same_bits():
    a = workloads.canvas_qkv(SMALL, 1)
    b = workloads.canvas_qkv(SMALL, 1)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    c = workloads.canvas_qkv(SMALL, 2)
    assert not torch.equal(a[0], c[0])                    # steps draw fresh tensors


def test_shapes_and_dtypes():
    w = SMALL
    q, kc, vc = workloads.canvas_qkv(w, 0)
    assert q.shape == (w.batch, w.canvas, w.heads_q, w.head_dim) and q.dtype == torch.bfloat16
    assert kc.shape == vc.shape == (w.batch, w.canvas, w.heads_kv, w.head_dim)
    kp, vp, cu = workloads.prefix_kv(w)
    assert kp.shape == (300, w.heads_kv, w.head_dim) and cu.tolist() == [0, 300]
    lg = workloads.logits(w, 0)
    assert lg.shape == (w.rows, w.vocab)


def test_logit_spike_is_the_row_maximum_mostly():
    """N(0, 3^2) plus 8 at one index per row: the spiked entry is the row's
    largest for most rows (the spike sits about 2.7 standard deviations up)."""
    w = SMALL
    lg = workloads.logits(w, 0).float()
    g = workloads._gen(w, "spike", 0, "cpu")
    idx = torch.randint(0, w.vocab, (w.rows,), generator=g)
    frac = (lg.argmax(dim=1) == idx).float().mean().item()
    assert frac > 0.2
    z = lg.clone()
    z[torch.arange(w.rows), idx] -= w.spike
    assert abs(z.std().item() - w.logit_std) < 0.05 * w.logit_std


def test_e4m3_factors_cover_the_tensors_they_scale():
    w = SMALL
    qs, kcs, vcs, kp, vp, cu, f = workloads.e4m3_block_inputs(w)
    assert qs.dtype == torch.float8_e4m3fn and qs.shape[0] == w.steps
    fk, fv = f[0][1], f[0][2]
    assert all(s[1] == fk and s[2] == fv for s in f)      # one K and one V factor per block
    assert all(_is_pow2(x) for s in f for x in s)
    f32 = dataclasses.replace(w, dtype="f32")
    kp32, vp32, _ = workloads.prefix_kv(f32)
    amax_k = max([kp32.abs().max().item()] +
                 [workloads.canvas_qkv(f32, s)[1].abs().max().item() for s in range(w.steps)])
    assert amax_k / fk <= 448.0 < 2 * amax_k / fk          # the smallest power of two that fits
    for s in range(w.steps):
        q8, _, _, _, _, _, fs = workloads.e4m3_attn_inputs(w, s)
        assert fs[0] == f[s][0]
        assert torch.equal(q8.view(torch.uint8), qs[s].view(torch.uint8))
    # decoded values are the float32 draws rounded to E4M3 (3 mantissa bits)
    dec = kp.float() * fk
    rel = ((dec - kp32).abs() / kp32.abs().clamp_min(fk * 2.0 ** -6)).max().item()
    assert rel <= 2.0 ** -4 + 1e-7
