"""The oracle: a plain float64 CPU implementation of one denoising step of
block discrete-diffusion decoding.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product library (``block_discrete_diffusion_dd_b200``) never imports,
links or calls anything here, and this package imports nothing from it.

The arithmetic lives in ``dd_oracle.c`` (plain C, float64, one OpenMP loop
over independent rows); this module only marshals numpy arrays and runs the
step loop of a block in plain Python.

Sources: "DiffusionGemma Technical Report" (paperfeed review), sections "The
mechanism: an AR model turned inside out" and "Training"; Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3" (SC'11) for Philox4x32-10.

Parity status per function (what pins it; tests/test_oracle_*.py):
  philox4x32_10 / words     -- torch's independent CPU Philox engine
                               (ATen PhiloxRNGEngine), bit-exact; uniformity.
  canvas_attn               -- float64 torch SDPA, pure-Python brute force,
                               closed forms, permutation/zero-prefix/GQA
                               invariants.
  e4m3_value / E4M3 inputs  -- closed-form codes of the OCP E4M3 encoding,
                               torch's float8_e4m3fn decoding of all 256
                               codes; E4M3 attention with power-of-two
                               per-tensor factors equals the float32 path on
                               the exactly scaled values.
  sample_renoise            -- chi-square of Gumbel-max vs softmax, scipy
                               log-softmax/entropy, spike and constant-logit
                               closed forms, binomial re-noise rate,
                               chi-square uniformity of replacements.
  init_canvas               -- chi-square uniformity; shares the replacement
                               rule pinned above.
  denoise_block             -- a loop of the two pinned functions (plain
                               Python), checked for step0-restart identity.
  entropy_accept / stop_check -- greedy budgeted-prefix properties, closed
                               forms, ties, the strict threshold.
  denoise_block_adaptive    -- a loop of the pinned sampler, halt test and
                               acceptance (plain Python); closed cases built
                               so every step's outcome is known: a halt at
                               a chosen step, two canvases halting at
                               different steps with the first frozen, no
                               halt within max_steps.
  soft_embed                -- pure-Python brute force, closed forms
                               (constant logits -> mean embedding, one
                               dominant logit -> its embedding row),
                               temperature scaling, linearity in E.
  ffw / self_condition      -- pure-Python brute force with math.erf,
                               tabulated values of the normal distribution
                               function, closed forms (zero weights, large
                               arguments), linearity in W2 and b2.

Regression fixtures: tests/golden/*.json, written from this package alone by
tests/golden/make_golden.py (the pages print no worked example), freeze its
outputs on small inputs; tests/test_golden_cpu.py checks that they still
hold.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16 = 0
F32 = 1
E4M3 = 2

_lib = None


def build(force: bool = False) -> str:
    """Compile dd_oracle.c with gcc (float64, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32, i64, u32, u64, f64, f32 = (ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                    ctypes.c_uint64, ctypes.c_double, ctypes.c_float)
    lib.oracle_word.restype = u32
    lib.oracle_word.argtypes = [u64, u32, u32, u32, u32]
    lib.oracle_uniform.restype = f64
    lib.oracle_uniform.argtypes = [u32]
    lib.oracle_words.restype = None
    lib.oracle_words.argtypes = [u64, u32, u32, P, P, i64, P]
    lib.oracle_philox_blocks.restype = None
    lib.oracle_philox_blocks.argtypes = [P, P, i64, P]
    lib.oracle_canvas_attn.restype = i32
    lib.oracle_canvas_attn.argtypes = [i32, i32, i32, i32, i32, f64, i32, P, P, P, P, P, P, P, P,
                                       i32, P, P, i32]
    lib.oracle_e4m3_value.restype = f64
    lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.oracle_sample_renoise.restype = i32
    lib.oracle_sample_renoise.argtypes = [P, i32, i64, i64, i64, P, i64, f64, f32, u64, u32, u32,
                                          P, P, P, P, P, P, P, i32]
    lib.oracle_init_canvas.restype = None
    lib.oracle_init_canvas.argtypes = [P, i64, i64, u64, u32]
    lib.oracle_entropy_accept.argtypes = [P, P, i64, i64, f64, u64, u32, u32, i64, P, P, P, P]
    lib.oracle_entropy_accept.restype = None
    lib.oracle_stop_check.argtypes = [P, P, P, i64, i64, f64, P]
    lib.oracle_stop_check.restype = None
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _raw(x):
    """(numpy array, dtype code) from a torch tensor or numpy array.

    bf16 and E4M3 tensors are passed as their raw 16- and 8-bit patterns; the
    C side decodes them exactly.  Anything else must already be float32.
    """
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)), BF16
            if x.dtype == torch.float8_e4m3fn:
                return np.ascontiguousarray(x.view(torch.uint8).numpy()), E4M3
            if x.dtype == torch.float32:
                return np.ascontiguousarray(x.numpy()), F32
            raise TypeError(f"oracle: unsupported tensor dtype {x.dtype}")
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), BF16
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), F32
    raise TypeError(f"oracle: unsupported array dtype {x.dtype}")


# ---------------------------------------------------------------- Philox

def philox4x32_10(ctrs, keys):
    """Philox4x32-10 blocks: ctrs [n,4] uint32, keys [n,2] uint32 -> [n,4]."""
    lib = _load()
    c = np.ascontiguousarray(ctrs, dtype=np.uint32).reshape(-1, 4)
    k = np.ascontiguousarray(keys, dtype=np.uint32).reshape(-1, 2)
    assert c.shape[0] == k.shape[0]
    out = np.empty_like(c)
    lib.oracle_philox_blocks(_ptr(c), _ptr(k), c.shape[0], _ptr(out))
    return out


def words(seed: int, stream: int, step: int, rows, vs):
    """32-bit words for counter (v >> 2, row, step, stream), word v & 3."""
    lib = _load()
    r = np.ascontiguousarray(rows, dtype=np.uint32).ravel()
    v = np.ascontiguousarray(vs, dtype=np.uint32).ravel()
    assert r.shape == v.shape
    out = np.empty_like(r)
    lib.oracle_words(seed, stream, step, _ptr(r), _ptr(v), r.size, _ptr(out))
    return out


def uniform(x: int) -> float:
    return _load().oracle_uniform(int(x))


# ------------------------------------------------------- canvas attention

def e4m3_value(code: int) -> float:
    """The value of one E4M3 byte (OCP OFP8 E4M3 encoding)."""
    return _load().oracle_e4m3_value(int(code) & 0xFF)


def canvas_attn(q, kc, vc, kp, vp, cu_prefix, scale=None, positions=None, threads=0,
                qkv_scale=None):
    """float64 attention over [prefix_b || canvas_b] for every (b, i, h).

    Shapes: q [B,C,Hq,D]; kc, vc [B,C,Hkv,D]; kp, vp [sum L_b, Hkv, D];
    cu_prefix [B+1] int.  positions: optional list of canvas positions to
    compute (others are NaN).  qkv_scale: optional per-tensor factors
    (q, k, v) multiplying the stored values (8-bit inputs with per-tensor
    scales).  Returns (out [B,C,Hq,D], lse [B,Hq,C]).
    """
    lib = _load()
    qa, dt = _raw(q)
    kca, dt2 = _raw(kc)
    vca, dt3 = _raw(vc)
    kpa, dt4 = _raw(kp)
    vpa, dt5 = _raw(vp)
    if len({dt, dt2, dt3, dt4, dt5}) != 1:
        raise TypeError("oracle: mixed input dtypes")
    B, C, Hq, D = qa.shape
    Hkv = kca.shape[2]
    cu = np.ascontiguousarray(np.asarray(cu_prefix, dtype=np.int32))
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.full((B, C, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((B, Hq, C), np.nan, dtype=np.float64)
    if positions is None:
        pos, npos = None, -1
    else:
        pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int32))
        npos = pos.size
    sc = None if qkv_scale is None else np.ascontiguousarray(np.asarray(qkv_scale, np.float64))
    if sc is not None and sc.shape != (3,):
        raise ValueError("oracle: qkv_scale must hold three factors")
    rc = lib.oracle_canvas_attn(B, C, Hq, Hkv, D, float(scale), dt, _ptr(sc), _ptr(qa), _ptr(kca),
                                _ptr(vca), _ptr(kpa), _ptr(vpa), _ptr(cu), _ptr(pos), npos,
                                _ptr(out), _ptr(lse), int(threads))
    if rc != 0:
        raise ValueError("oracle_canvas_attn: bad arguments")
    return out, lse


# ------------------------------------------------------------------ sampler

def sample_renoise(logits, tau, rate, seed, step, row_offset=0, rows=None, row_stride=None,
                   vocab=None, n_rows=None, threads=0):
    """One sampler step (Gumbel-max, confidence, entropy, re-noise).

    logits: [R, V] (bf16 or f32).  rows: optional local row indices to compute.
    row_stride/vocab/n_rows override the shape (row_stride 0 broadcasts one
    row to n_rows rows).  Returns a dict of numpy arrays indexed like `rows`.
    """
    lib = _load()
    la, dt = _raw(logits)
    if vocab is None:
        vocab = la.shape[-1]
    if row_stride is None:
        row_stride = la.shape[-1]
    if n_rows is None:
        n_rows = la.size // la.shape[-1]
    if rows is None:
        sel, nsel = None, -1
        n = n_rows
    else:
        sel = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nsel = sel.size
        n = nsel
    res = {
        "tokens": np.empty(n, np.int32), "pred": np.empty(n, np.int32),
        "conf": np.empty(n, np.float64), "entropy": np.empty(n, np.float64),
        "renoised": np.empty(n, np.uint8), "gap": np.empty(n, np.float64),
        "best": np.empty(n, np.float64),
    }
    rc = lib.oracle_sample_renoise(
        _ptr(la), dt, int(n_rows), int(vocab), int(row_stride), _ptr(sel), int(nsel), float(tau),
        float(np.float32(rate)), int(seed), int(step), int(row_offset), _ptr(res["tokens"]),
        _ptr(res["pred"]), _ptr(res["conf"]), _ptr(res["entropy"]), _ptr(res["renoised"]),
        _ptr(res["gap"]), _ptr(res["best"]), int(threads))
    if rc != 0:
        raise ValueError("oracle_sample_renoise: bad arguments")
    return res


def init_canvas(rows: int, vocab: int, seed: int, row_offset: int = 0):
    lib = _load()
    out = np.empty(rows, np.int32)
    lib.oracle_init_canvas(_ptr(out), rows, vocab, seed, row_offset)
    return out


# ------------------------------------------------ the pages' sampler policy

def anneal_temperature(s: int, steps: int, t0: float = 0.8, t1: float = 0.4) -> float:
    """Temperature of step s of a block whose nominal budget is `steps`:
    annealed linearly from t0 to t1 ("The mechanism", sampler paragraph:
    tau 0.8 -> 0.4; the pages give the end points only, linear in the step
    index over the nominal budget is the reading taken), as float32."""
    if steps <= 1:
        return float(np.float32(t0))
    return float(np.float32(t0 + (t1 - t0) * s / (steps - 1)))


def entropy_accept(entropy, pred, canvas: int, budget: float, seed: int, step: int, vocab: int,
                   row_offset: int = 0):
    """Entropy-budget acceptance (dd_oracle.c: oracle_entropy_accept).

    entropy: float32 [B*C] (rounded to float32 here), pred int32 [B*C].
    Returns dict(tokens, accepted, n_accepted [B], sum_accepted [B])."""
    lib = _load()
    h = np.ascontiguousarray(np.asarray(entropy, dtype=np.float32).reshape(-1))
    pr = np.ascontiguousarray(np.asarray(pred, dtype=np.int32).reshape(-1))
    assert h.size == pr.size and h.size % canvas == 0
    B = h.size // canvas
    res = {"tokens": np.empty(h.size, np.int32), "accepted": np.empty(h.size, np.uint8),
           "n_accepted": np.empty(B, np.int32), "sum_accepted": np.empty(B, np.float64)}
    lib.oracle_entropy_accept(_ptr(h), _ptr(pr), B, canvas, float(budget), int(seed), int(step),
                              int(row_offset), int(vocab), _ptr(res["tokens"]),
                              _ptr(res["accepted"]), _ptr(res["n_accepted"]),
                              _ptr(res["sum_accepted"]))
    return res


def stop_check(entropy, pred, pred_prev, canvas: int, threshold: float = 0.005):
    """Early-halt test per canvas (dd_oracle.c: oracle_stop_check)."""
    lib = _load()
    h = np.ascontiguousarray(np.asarray(entropy, dtype=np.float32).reshape(-1))
    pr = np.ascontiguousarray(np.asarray(pred, dtype=np.int32).reshape(-1))
    pp = None if pred_prev is None else np.ascontiguousarray(
        np.asarray(pred_prev, dtype=np.int32).reshape(-1))
    B = h.size // canvas
    done = np.empty(B, np.uint8)
    lib.oracle_stop_check(_ptr(h), _ptr(pr), _ptr(pp), B, canvas, float(threshold), _ptr(done))
    return done


def _acceptance_margin(h32: np.ndarray, budget: float) -> float:
    """How far one canvas's acceptance is from flipping: the distance of the
    budget to the float64 running sum on either side of the cut, and the gap
    between the last accepted and the first rejected entropy (a smaller
    perturbation of the entropies cannot change the accepted set)."""
    order = np.lexsort((np.arange(h32.size), h32))     # entropy, then position
    hs = [float(x) for x in h32[order]]
    total, k = 0.0, 0
    while k < len(hs) and total + hs[k] <= budget:     # the acceptance walk
        total += hs[k]
        k += 1
    m = np.inf
    if k > 0:
        m = min(m, budget - total)
    if k < len(hs):
        m = min(m, total + hs[k] - budget)
        if k > 0:
            m = min(m, hs[k] - hs[k - 1])
    return float(m)


def denoise_block_adaptive(logits_steps, temperatures, budget: float, stop_entropy: float,
                           seed: int, canvas: int, max_steps=None, step0: int = 0,
                           init_canvas=None, threads: int = 0):
    """The pages' adaptive block loop ("DiffusionGemma Technical Report"
    (paperfeed review), "The mechanism", sampler paragraph): per step, the
    sampler at that step's temperature with no scheduled re-noise, the halt
    test (low mean entropy and the same prediction as the previous step),
    then the entropy-budget acceptance.  Readings: a canvas that halts at
    step s takes its step-s prediction everywhere and later steps leave it
    alone; the loop ends once every canvas has halted, or after max_steps.

    The sampler's entropies are rounded to float32 (the precision the step
    outputs them in) before the halt test and the acceptance, which sum
    them in float64.  Composed in plain Python from sample_renoise,
    stop_check and entropy_accept, each pinned on its own.

    logits_steps: [S, B*canvas, V] (bf16 or float32).  Returns a dict:
      canvas [B*C], history [steps_run, B*C], halt_step [B] (-1 = never),
      steps_run, and per step (lists of [B] arrays) the margins of its
      decisions, for telling a genuine mismatch from a near-boundary one:
      min_gap (smallest top-two Gumbel score gap in the canvas),
      stop_margin (|mean entropy - stop_entropy|), accept_margin
      (_acceptance_margin), plus pred and entropy (float32) per step.
    """
    S = len(logits_steps) if max_steps is None else int(max_steps)
    R = int(logits_steps[0].shape[0])
    assert R % canvas == 0
    B = R // canvas
    cur = (np.zeros(R, np.int32) if init_canvas is None
           else np.asarray(init_canvas, np.int32).copy())
    done = np.zeros(B, bool)
    halt = np.full(B, -1, np.int32)
    prev = None
    out = {"history": [], "min_gap": [], "stop_margin": [], "accept_margin": [], "pred": [],
           "entropy": []}
    steps_run = 0
    for s in range(S):
        r = sample_renoise(logits_steps[s], temperatures[s], 0.0, seed, step0 + s,
                           threads=threads)
        pred = r["pred"]
        h32 = r["entropy"].astype(np.float32)
        now = stop_check(h32, pred, prev, canvas, stop_entropy).astype(bool) & ~done
        acc = entropy_accept(h32, pred, canvas, budget, seed, step0 + s, int(
            logits_steps[s].shape[-1]))
        gap, stop_m, acc_m = (np.empty(B) for _ in range(3))
        for b in range(B):
            sl = slice(b * canvas, (b + 1) * canvas)
            gap[b] = r["gap"][sl].min()
            stop_m[b] = abs(h32[sl].astype(np.float64).sum() / canvas - stop_entropy)
            acc_m[b] = _acceptance_margin(h32[sl], budget)
            if done[b]:
                continue                        # halted at an earlier step: frozen
            if now[b]:
                cur[sl] = pred[sl]              # halts now: its whole prediction
                halt[b] = s
            else:
                cur[sl] = acc["tokens"][sl]
        done |= now
        out["history"].append(cur.copy())
        out["min_gap"].append(gap)
        out["stop_margin"].append(stop_m)
        out["accept_margin"].append(acc_m)
        out["pred"].append(pred)
        out["entropy"].append(h32)
        prev = pred
        steps_run = s + 1
        if done.all():
            break
    out.update(canvas=cur, halt_step=halt, steps_run=steps_run,
               history=np.stack(out["history"]) if out["history"] else np.zeros((0, R), np.int32))
    return out


# ---------------------------------------- self-conditioning soft embedding

def _f64(x) -> np.ndarray:
    """float64 copy of a bf16 or float32 tensor / array (exact decoding)."""
    a, dt = _raw(x)
    if dt == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def soft_embed(logits, tau: float, emb, rows=None, cols=None, v_chunk: int = 16384):
    """The self-conditioning signal before its MLP ("DiffusionGemma Technical
    Report" (paperfeed review), "The mechanism", self-conditioning
    paragraph): the step's predicted token distribution of each position,
    p0 = softmax(logits / tau) (the distribution the sampler draws from),
    pushed through the embedding matrix E:
        out[r, :] = sum_v p0[r, v] E[v, :].
    Plain float64: logits [R, V] and E [V, d] (bf16 or float32, decoded
    exactly); the softmax with its row maximum subtracted; the sum over v in
    chunks of v_chunk (a plain matrix product per chunk).  rows / cols
    restrict the output rows / embedding columns computed."""
    lg = _f64(logits)
    if rows is not None:
        lg = lg[np.asarray(rows)]
    z = lg / float(tau)
    z -= z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    e_raw, e_dt = _raw(emb)
    if cols is not None:
        e_raw = e_raw[:, np.asarray(cols)]
    out = np.zeros((p.shape[0], e_raw.shape[1]), np.float64)
    for v0 in range(0, p.shape[1], v_chunk):
        blk = e_raw[v0:v0 + v_chunk]
        e = ((blk.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if e_dt == BF16
             else blk.astype(np.float64))
        out += p[:, v0:v0 + v_chunk] @ e
    return out


def _gelu64(x: np.ndarray) -> np.ndarray:
    """GELU(x) = x * Phi(x) = x (1 + erf(x / sqrt 2)) / 2, float64 (erf from
    torch's float64 CPU routine)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    return (0.5 * t * (1.0 + torch.erf(t / np.sqrt(2.0)))).numpy()


def ffw(u, w1, b1, w2, b2) -> np.ndarray:
    """The self-conditioning MLP ("DiffusionGemma Technical Report"
    (paperfeed review), "The mechanism", self-conditioning paragraph:
    z_t = FFW(p0 E), a small MLP of 7.8M parameters).  The pages give no
    architecture; read as two dense layers with a GELU between them:
        z = GELU(u W1 + b1) W2 + b2
    in float64 from the exactly decoded bf16 / float32 inputs: u [rows, d],
    W1 [d, h], b1 [h], W2 [h, d], b2 [d]."""
    h = _gelu64(_f64(u) @ _f64(w1) + _f64(b1))
    return h @ _f64(w2) + _f64(b2)


def self_condition(logits, tau: float, emb, w1, b1, w2, b2) -> np.ndarray:
    """z = FFW(softmax(logits / tau) E): soft_embed followed by ffw, both in
    float64 (no rounding in between)."""
    u = soft_embed(logits, tau, emb)
    h = _gelu64(u @ _f64(w1) + _f64(b1))
    return h @ _f64(w2) + _f64(b2)


# --------------------------------------------------------- the block loop

def denoise_block(steps, q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps, rates,
                  temperatures, seed, step0=0, scale=None, positions=None, sample_rows=None,
                  threads=0):
    """The step loop of one block: for s in 0..S-1, attention of step s and
    the sampler of step s (Philox step = step0 + s).  The sampler does not
    read the previous canvas: each step's canvas is its pred-or-replacement.

    Returns (attn_out list, lse list, per-step sampler dicts).
    """
    outs, lses, samp = [], [], []
    for s in range(steps):
        if q_steps is not None:
            o, l = canvas_attn(q_steps[s], kc_steps[s], vc_steps[s], kp, vp, cu_prefix, scale,
                               positions, threads)
            outs.append(o)
            lses.append(l)
        samp.append(sample_renoise(logits_steps[s], temperatures[s], rates[s], seed, step0 + s,
                                   0, sample_rows, threads=threads))
    return outs, lses, samp
