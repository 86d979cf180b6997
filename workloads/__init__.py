"""Seeded synthetic inputs for the denoise-step workloads.

This module holds shapes, distributions and seeds only: none of the method's
arithmetic.  Both sides of every parity check (the CUDA library and the
float64 oracle) consume the tensors it makes, so it imports neither.

The five workloads mirror the shapes the method runs at ("DiffusionGemma
Technical Report", paperfeed review: 256-token canvas; 262,144-entry vocabulary
in "The numbers, honestly"; ~12 passes per block in "The mechanism"):

  tiny_fp32      B=1, Hq=2, Hkv=1, D=64, prefix 128, canvas 256, fp32, scale
                 1/8; sampler 256 x 1024 fp32 logits ~ N(0, 2^2), tau 1,
                 rate 0.5.
  b1_L4096       B=1, Hq=16, Hkv=8, D=128, prefix 4096, bf16; logits
                 256 x 262144 ~ N(0, 3^2) + 8 at one uniform index per row,
                 rate 0.3.
  long_L65536    as b1_L4096 with prefix 65536, rate 0.1.
  ragged_b8      B=8, prefix lengths numpy default_rng(0).integers(512, 16385,
                 8), logits 2048 x 262144, rate 0.2.
  block12_L8192  B=1, prefix 8192, 12 steps, fresh canvas Q/K/V and logits
                 per step keyed on (seed, step), rate_s = 0.9 (11 - s) / 11,
                 tau 1.

Every tensor is drawn in float32 from a torch.Generator seeded with a hash
of (seed, workload, tensor name, step), then rounded to bf16 (round to
nearest even) where the workload is bf16.  The 8-bit attention inputs are
the same float32 draws rounded to E4M3 under a power-of-two per-tensor
factor (e4m3_attn_inputs; e4m3_block_inputs for a block of steps).  The
generator's device is the
caller's choice; the same device always gives the same bits.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    canvas: int
    heads_q: int
    heads_kv: int
    head_dim: int
    prefix_lens: tuple
    dtype: str            # "f32" or "bf16"
    vocab: int
    logit_std: float
    spike: float           # added at one uniform index per row (0: none)
    rates: tuple           # one per step
    temperatures: tuple    # one per step
    steps: int = 1
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.head_dim))

    @property
    def rows(self) -> int:
        return self.batch * self.canvas

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def cu_prefix(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.prefix_lens)]).astype(np.int32)

    def attn_flops(self) -> int:
        """Algorithmic attention FLOPs of one step: 4 Hq C (L_b + C) D per row b."""
        return sum(4 * self.heads_q * self.canvas * (L + self.canvas) * self.head_dim
                   for L in self.prefix_lens)

    def logit_bytes(self) -> int:
        return self.rows * self.vocab * (4 if self.dtype == "f32" else 2)


def _ragged_lens():
    return tuple(int(x) for x in np.random.default_rng(0).integers(512, 16385, 8))


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 2, 1, 64, (128,), "f32", 1024, 2.0, 0.0,
                          (0.5,), (1.0,)),
    "b1_L4096": Workload("b1_L4096", 1, 256, 16, 8, 128, (4096,), "bf16", 262144, 3.0, 8.0,
                         (0.3,), (1.0,)),
    "long_L65536": Workload("long_L65536", 1, 256, 16, 8, 128, (65536,), "bf16", 262144, 3.0,
                            8.0, (0.1,), (1.0,)),
    "ragged_b8": Workload("ragged_b8", 8, 256, 16, 8, 128, _ragged_lens(), "bf16", 262144, 3.0,
                          8.0, (0.2,), (1.0,)),
    "block12_L8192": Workload("block12_L8192", 1, 256, 16, 8, 128, (8192,), "bf16", 262144, 3.0,
                              8.0, tuple(float(np.float32(0.9 * (11 - s) / 11)) for s in range(12)),
                              (1.0,) * 12, steps=12),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(w, **changes)


def _seed_for(w: Workload, tensor: str, step: int) -> int:
    h = hashlib.sha256(f"{w.seed}/{w.name}/{tensor}/{step}".encode()).hexdigest()
    return int(h[:15], 16)


def _gen(w: Workload, tensor: str, step: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed_for(w, tensor, step))
    return g


def _normal(w, tensor, step, shape, std, device):
    g = _gen(w, tensor, step, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(w.torch_dtype)


def canvas_qkv(w: Workload, step: int = 0, device="cpu", q_gain: float = 1.0):
    """Q [B,C,Hq,D], Kc, Vc [B,C,Hkv,D] for one step, i.i.d. N(0,1).

    q_gain > 1 scales Q before rounding (a sharper softmax that exercises the
    running-max rescale path)."""
    B, C, Hq, Hkv, D = w.batch, w.canvas, w.heads_q, w.heads_kv, w.head_dim
    q = _normal(w, "q", step, (B, C, Hq, D), q_gain, device)
    kc = _normal(w, "kc", step, (B, C, Hkv, D), 1.0, device)
    vc = _normal(w, "vc", step, (B, C, Hkv, D), 1.0, device)
    return q, kc, vc


def prefix_kv(w: Workload, device="cpu"):
    """Packed prefix cache Kp, Vp [sum L_b, Hkv, D] and cu_prefix [B+1]."""
    n = int(sum(w.prefix_lens))
    kp = _normal(w, "kp", 0, (n, w.heads_kv, w.head_dim), 1.0, device)
    vp = _normal(w, "vp", 0, (n, w.heads_kv, w.head_dim), 1.0, device)
    return kp, vp, torch.from_numpy(w.cu_prefix)


def to_e4m3(xs):
    """Round float32 tensors that share one scale factor to E4M3.

    The factor is the power of two f = 2^ceil(log2(amax / 448)) over all of
    them (448 = the largest finite E4M3 value), so x / f is exact in float32
    and never overflows; torch rounds x / f to the nearest E4M3 value (ties
    to even).  Returns (list of float8_e4m3fn tensors, f)."""
    amax = max(float(x.abs().max()) for x in xs if x.numel()) if any(x.numel() for x in xs) else 0.0
    f = 2.0 ** math.ceil(math.log2(amax / 448.0)) if amax > 0 else 1.0
    return [(x / f).to(torch.float8_e4m3fn) for x in xs], f


def e4m3_attn_inputs(w: Workload, step: int = 0, device="cpu", q_gain: float = 1.0):
    """The attention inputs of `w` drawn as for bf16 (same seeds, float32
    normals), then rounded to E4M3 with one factor for Q, one shared by Kp and
    Kc, one shared by Vp and Vc.  Returns q, kc, vc, kp, vp (float8_e4m3fn),
    cu_prefix and the factors (f_q, f_k, f_v)."""
    f32 = dataclasses.replace(w, dtype="f32")
    q, kc, vc = canvas_qkv(f32, step, device, q_gain)
    kp, vp, cu = prefix_kv(f32, device)
    (q8,), fq = to_e4m3([q])
    (kc8, kp8), fk = to_e4m3([kc, kp])
    (vc8, vp8), fv = to_e4m3([vc, vp])
    return q8, kc8, vc8, kp8, vp8, cu, (fq, fk, fv)


def e4m3_block_inputs(w: Workload, device="cpu"):
    """The attention inputs of every step of `w` in E4M3, for the block loop.

    The prefix cache is fixed across steps while one K factor (and one V
    factor) covers the prefix and the step's canvas keys in a call, so the K
    factor is taken over Kp and every step's Kc together (likewise V); Q
    gets its own factor per step.  Returns q_steps [S,B,C,Hq,D], kc_steps,
    vc_steps [S,B,C,Hkv,D] (float8_e4m3fn), kp, vp, cu_prefix and the list
    of per-step factors (f_q[s], f_k, f_v)."""
    f32 = dataclasses.replace(w, dtype="f32")
    steps = [canvas_qkv(f32, s, device) for s in range(w.steps)]
    kp, vp, cu = prefix_kv(f32, device)
    (kp8, *kcs), fk = to_e4m3([kp] + [x[1] for x in steps])
    (vp8, *vcs), fv = to_e4m3([vp] + [x[2] for x in steps])
    qs, fq = zip(*(to_e4m3([x[0]]) for x in steps))

    def stack(ts):
        return torch.stack([t.view(torch.uint8) for t in ts]).view(torch.float8_e4m3fn)

    return (stack([q[0] for q in qs]), stack(kcs), stack(vcs), kp8, vp8, cu,
            [(f, fk, fv) for f in fq])


def logits(w: Workload, step: int = 0, device="cpu", rows: Optional[int] = None):
    """Logits [R, V]: N(0, std^2) plus `spike` at one uniform index per row."""
    R = w.rows if rows is None else rows
    g = _gen(w, "logits", step, device)
    x = torch.randn((R, w.vocab), generator=g, device=device, dtype=torch.float32)
    x.mul_(w.logit_std)
    if w.spike:
        gi = _gen(w, "spike", step, device)
        idx = torch.randint(0, w.vocab, (R,), generator=gi, device=device)
        x[torch.arange(R, device=device), idx] += w.spike
    return x.to(w.torch_dtype)


def embedding(w: Workload, d: Optional[int] = None, device="cpu"):
    """A synthetic embedding matrix E [V, d], i.i.d. N(0, 1), in the
    workload's dtype.  d defaults to Hq * D, the model width the attention
    geometry implies (the pages do not state it)."""
    d = w.heads_q * w.head_dim if d is None else d
    return _normal(w, "embedding", 0, (w.vocab, d), 1.0, device)


# Hidden width of the self-conditioning MLP: the pages give only its size
# (7.8M parameters).  Two dense layers d -> h -> d with biases at d = 2048
# and h = 1904 hold 2 * 2048 * 1904 + 1904 + 2048 = 7,802,784 parameters.
FFW_HIDDEN = 1904


def ffw_weights(w: Workload, d: Optional[int] = None, hidden: int = FFW_HIDDEN, device="cpu"):
    """Synthetic weights of the self-conditioning MLP in the workload's
    dtype: W1 [d, h] ~ N(0, 1/d), b1 [h] ~ N(0, 0.1^2), W2 [h, d] ~ N(0, 1/h),
    b2 [d] ~ N(0, 0.1^2) (fan-in scaling keeps the activations of order 1)."""
    d = w.heads_q * w.head_dim if d is None else d
    w1 = _normal(w, "ffw_w1", 0, (d, hidden), 1.0 / math.sqrt(d), device)
    b1 = _normal(w, "ffw_b1", 0, (hidden,), 0.1, device)
    w2 = _normal(w, "ffw_w2", 0, (hidden, d), 1.0 / math.sqrt(hidden), device)
    b2 = _normal(w, "ffw_b2", 0, (d,), 0.1, device)
    return w1, b1, w2, b2


def ffw_input(w: Workload, rows: Optional[int] = None, d: Optional[int] = None, device="cpu"):
    """A synthetic MLP input u [rows, d] ~ N(0, 1) (standing in for p0 E)."""
    d = w.heads_q * w.head_dim if d is None else d
    rows = w.rows if rows is None else rows
    return _normal(w, "ffw_u", 0, (rows, d), 1.0, device)


def all_steps(w: Workload, device="cpu"):
    """Per-step canvas Q/K/V and logits for every step of the workload."""
    qs, kcs, vcs, ls = [], [], [], []
    for s in range(w.steps):
        q, kc, vc = canvas_qkv(w, s, device)
        qs.append(q)
        kcs.append(kc)
        vcs.append(vc)
        ls.append(logits(w, s, device))
    return torch.stack(qs), torch.stack(kcs), torch.stack(vcs), torch.stack(ls)


def names() -> List[str]:
    return list(WORKLOADS)
