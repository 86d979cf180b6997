"""Python binding of libdd, the B200 (sm_100a) library for one denoising step
of block discrete-diffusion decoding ("DiffusionGemma Technical Report",
paperfeed review, "The mechanism: an AR model turned inside out").

This module only marshals arguments: torch tensors in, raw device pointers
and sizes out to the C ABI (include/dd.h); torch provides device memory and
streams.  Every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: if libdd.so is missing or the GPU is unusable,
calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdd.so")

DD_BF16, DD_F32, DD_E4M3 = 0, 1, 2
STATUS = {0: "DD_OK", 1: "DD_ERR_INVALID_ARG", 2: "DD_ERR_UNSUPPORTED", 3: "DD_ERR_WORKSPACE",
          4: "DD_ERR_CUDA", 5: "DD_ERR_DEVICE_TIMEOUT", 6: "DD_ERR_DEVICE_BOUNDS"}

# every symbol include/dd.h declares
EXPORTS = (
    "dd_canvas_attn_workspace", "dd_canvas_attn", "dd_sample_renoise_workspace",
    "dd_sample_renoise", "dd_init_canvas", "dd_denoise_block_workspace", "dd_denoise_block",
    "dd_workspace_init", "dd_query_device_error", "dd_status_string", "dd_last_error",
    "dd_launch_count", "dd_reset_launch_count", "dd_sample_renoise_noalloc",
    "dd_entropy_accept", "dd_stop_check", "dd_denoise_block_adaptive_workspace",
    "dd_denoise_block_adaptive", "dd_canvas_attn_fp8", "dd_denoise_block_graph_create",
    "dd_denoise_block_graph_launch", "dd_denoise_block_graph_destroy",
    "dd_soft_embed_workspace", "dd_soft_embed", "dd_denoise_block_fp8",
    "dd_denoise_block_adaptive_graph_create", "dd_denoise_block_adaptive_graph_launch",
    "dd_denoise_block_adaptive_graph_destroy", "dd_ffw_workspace", "dd_ffw",
    "dd_self_condition_workspace", "dd_self_condition", "dd_set_test_stall_ns",
)


class DDError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("canvas", ctypes.c_int), ("heads_q", ctypes.c_int),
                ("heads_kv", ctypes.c_int), ("head_dim", ctypes.c_int), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int)]


class Fp8Scales(ctypes.Structure):
    _fields_ = [("q", ctypes.c_float), ("k", ctypes.c_float), ("v", ctypes.c_float)]


class SampleParams(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("renoise_rate", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("step", ctypes.c_uint32),
                ("row_offset", ctypes.c_uint32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libdd.so (built in-tree by build.build()); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libdd.so not found at {LIB_PATH}: run "
                           "block_discrete_diffusion_dd_b200.build.build() first")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, u32, u64, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                 ctypes.c_uint64, ctypes.c_size_t)
    f32 = ctypes.c_float
    D = ctypes.POINTER(AttnDesc)
    lib.dd_canvas_attn_workspace.restype = sz
    lib.dd_canvas_attn_workspace.argtypes = [D, P]
    lib.dd_canvas_attn.restype = i32
    lib.dd_canvas_attn.argtypes = [D, P, P, P, P, P, P, P, P, P, P, sz, P]
    lib.dd_canvas_attn_fp8.restype = i32
    lib.dd_canvas_attn_fp8.argtypes = [D, P, P, P, P, P, P, P, ctypes.POINTER(Fp8Scales), P, P, P,
                                       sz, P]
    lib.dd_sample_renoise_workspace.restype = sz
    lib.dd_sample_renoise_workspace.argtypes = [i32, i32, i32]
    lib.dd_sample_renoise.restype = i32
    lib.dd_sample_renoise.argtypes = [P, i32, i32, i32, i64, ctypes.POINTER(SampleParams), P, P, P,
                                      P, P, P, sz, P]
    lib.dd_sample_renoise_noalloc.restype = i32
    lib.dd_sample_renoise_noalloc.argtypes = [P, i32, i32, i32, i64, ctypes.POINTER(SampleParams),
                                              P, P, P, P, P, P]
    lib.dd_init_canvas.restype = i32
    lib.dd_init_canvas.argtypes = [P, i32, i32, u64, u32, P]
    lib.dd_denoise_block_workspace.restype = sz
    lib.dd_denoise_block_workspace.argtypes = [D, P, i32]
    lib.dd_denoise_block.restype = i32
    lib.dd_denoise_block.argtypes = [D, i32, P, P, P, P, P, P, P, P, P, i32, P, P, u64, u32, P, P,
                                     P, P, sz, P]
    lib.dd_denoise_block_fp8.restype = i32
    lib.dd_denoise_block_fp8.argtypes = [D, i32, P, P, P, P, P, P, P, P, P, P, i32, P, P, u64, u32,
                                         P, P, P, P, sz, P]
    lib.dd_denoise_block_graph_create.restype = i32
    lib.dd_denoise_block_graph_create.argtypes = [ctypes.POINTER(P), D, i32, P, P, P, P, P, P, P,
                                                  P, P, i32, P, P, u64, u32, P, P, P, P, sz]
    lib.dd_denoise_block_graph_launch.restype = i32
    lib.dd_denoise_block_graph_launch.argtypes = [P, P]
    lib.dd_denoise_block_graph_destroy.restype = i32
    lib.dd_denoise_block_graph_destroy.argtypes = [P]
    lib.dd_denoise_block_adaptive_graph_create.restype = i32
    lib.dd_denoise_block_adaptive_graph_create.argtypes = [ctypes.POINTER(P), D, i32, P, P, P, P,
                                                           P, P, P, P, P, i32, P, f32, f32, u64,
                                                           u32, P, P, P, P, P, sz]
    lib.dd_denoise_block_adaptive_graph_launch.restype = i32
    lib.dd_denoise_block_adaptive_graph_launch.argtypes = [P, P]
    lib.dd_denoise_block_adaptive_graph_destroy.restype = i32
    lib.dd_denoise_block_adaptive_graph_destroy.argtypes = [P]
    lib.dd_soft_embed_workspace.restype = sz
    lib.dd_soft_embed_workspace.argtypes = [i32, i32, i32]
    lib.dd_soft_embed.restype = i32
    lib.dd_soft_embed.argtypes = [P, i32, i32, i32, i64, ctypes.c_float, P, i32, P, P, sz, P]
    lib.dd_set_test_stall_ns.restype = None
    lib.dd_set_test_stall_ns.argtypes = [u64]
    lib.dd_ffw_workspace.restype = sz
    lib.dd_ffw_workspace.argtypes = [i32, i32, i32]
    lib.dd_ffw.restype = i32
    lib.dd_ffw.argtypes = [P, i32, i32, i32, P, P, P, P, P, P, sz, P]
    lib.dd_self_condition_workspace.restype = sz
    lib.dd_self_condition_workspace.argtypes = [i32, i32, i32, i32]
    lib.dd_self_condition.restype = i32
    lib.dd_self_condition.argtypes = [P, i32, i32, i32, i64, ctypes.c_float, P, i32, P, P, i32, P,
                                      P, P, P, P, sz, P]
    lib.dd_entropy_accept.restype = i32
    lib.dd_entropy_accept.argtypes = [P, P, i32, i32, i32, f32, u64, u32, u32, P, P, P]
    lib.dd_stop_check.restype = i32
    lib.dd_stop_check.argtypes = [P, P, P, i32, i32, f32, ctypes.c_int32, P, P, P]
    lib.dd_denoise_block_adaptive_workspace.restype = sz
    lib.dd_denoise_block_adaptive_workspace.argtypes = [D, P, i32]
    lib.dd_denoise_block_adaptive.restype = i32
    lib.dd_denoise_block_adaptive.argtypes = [D, i32, P, P, P, P, P, P, P, P, P, i32, P, f32, f32,
                                              u64, u32, P, P, P, ctypes.POINTER(ctypes.c_int),
                                              P, sz, P]
    lib.dd_workspace_init.restype = i32
    lib.dd_workspace_init.argtypes = [P, sz, P]
    lib.dd_query_device_error.restype = i32
    lib.dd_query_device_error.argtypes = [P, P]
    lib.dd_status_string.restype = ctypes.c_char_p
    lib.dd_status_string.argtypes = [i32]
    lib.dd_last_error.restype = ctypes.c_char_p
    lib.dd_last_error.argtypes = []
    lib.dd_launch_count.restype = u64
    lib.dd_launch_count.argtypes = []
    lib.dd_reset_launch_count.restype = None
    lib.dd_reset_launch_count.argtypes = []
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        raise DDError(status, load().dd_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DD_BF16
    if t.dtype == torch.float32:
        return DD_F32
    if t.dtype == torch.float8_e4m3fn:
        return DD_E4M3
    raise TypeError(f"unsupported dtype {t.dtype} (bf16, fp32 or float8_e4m3fn)")


def _host_i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def new_workspace(nbytes: int, device=None, stream=None) -> torch.Tensor:
    """A device workspace (torch-owned) with its error word cleared."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    ws = torch.empty(max(int(nbytes), 256) + 256, dtype=torch.uint8, device=dev)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + max(int(nbytes), 256)]
    _check(load().dd_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))
    return ws


def attn_desc(q: torch.Tensor, kc: torch.Tensor, scale: Optional[float] = None) -> AttnDesc:
    B, C, Hq, D = q.shape
    Hkv = kc.shape[2]
    return AttnDesc(B, C, Hq, Hkv, D, float(scale if scale is not None else D ** -0.5),
                    _dtype_code(q))


def canvas_attn_workspace_bytes(desc: AttnDesc, cu_prefix_host) -> int:
    cu = _host_i32(cu_prefix_host)
    return int(load().dd_canvas_attn_workspace(ctypes.byref(desc), cu.ctypes.data_as(ctypes.c_void_p)))


def canvas_attn(q, kc, vc, kp, vp, cu_prefix, cu_prefix_host=None, scale=None, out=None,
                lse=None, want_lse=False, workspace=None, stream=None):
    """dd_canvas_attn: q [B,C,Hq,D], kc/vc [B,C,Hkv,D], kp/vp [sumL,Hkv,D],
    cu_prefix int32 [B+1] on the device.  Returns (out, lse or None)."""
    lib = load()
    desc = attn_desc(q, kc, scale)
    cu_h = _host_i32(cu_prefix if cu_prefix_host is None else cu_prefix_host)
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((desc.batch, desc.heads_q, desc.canvas), dtype=torch.float32,
                          device=q.device)
    if workspace is None:
        workspace = new_workspace(canvas_attn_workspace_bytes(desc, cu_h), q.device, stream)
    _check(lib.dd_canvas_attn(ctypes.byref(desc), _ptr(q), _ptr(kc), _ptr(vc), _ptr(kp), _ptr(vp),
                              _ptr(cu_prefix), cu_h.ctypes.data_as(ctypes.c_void_p), _ptr(out),
                              _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def canvas_attn_fp8(q, kc, vc, kp, vp, cu_prefix, scales, cu_prefix_host=None, scale=None,
                    out=None, lse=None, want_lse=False, workspace=None, stream=None):
    """dd_canvas_attn_fp8: float8_e4m3fn q [B,C,Hq,D], kc/vc [B,C,Hkv,D],
    kp/vp [sumL,Hkv,D]; scales = (f_q, f_k, f_v) per-tensor factors.
    Returns (out bf16 [B,C,Hq,D], lse or None)."""
    lib = load()
    desc = attn_desc(q, kc, scale)
    cu_h = _host_i32(cu_prefix if cu_prefix_host is None else cu_prefix_host)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if want_lse and lse is None:
        lse = torch.empty((desc.batch, desc.heads_q, desc.canvas), dtype=torch.float32,
                          device=q.device)
    if workspace is None:
        workspace = new_workspace(canvas_attn_workspace_bytes(desc, cu_h), q.device, stream)
    f = Fp8Scales(*(float(x) for x in scales))
    _check(lib.dd_canvas_attn_fp8(ctypes.byref(desc), _ptr(q), _ptr(kc), _ptr(vc), _ptr(kp),
                                  _ptr(vp), _ptr(cu_prefix), cu_h.ctypes.data_as(ctypes.c_void_p),
                                  ctypes.byref(f), _ptr(out), _ptr(lse), _ptr(workspace),
                                  workspace.numel(), _stream(stream)))
    return out, lse


def sample_workspace_bytes(rows: int, vocab: int, dtype=torch.bfloat16) -> int:
    code = DD_BF16 if dtype == torch.bfloat16 else DD_F32
    return int(load().dd_sample_renoise_workspace(rows, vocab, code))


def sample_renoise(logits: torch.Tensor, temperature: float, rate: float, seed: int, step: int,
                   row_offset: int = 0, rows: Optional[int] = None, vocab: Optional[int] = None,
                   row_stride: Optional[int] = None, outputs: Optional[dict] = None,
                   workspace=None, stream=None) -> dict:
    """dd_sample_renoise over logits [R, V] (bf16/fp32).  Returns a dict of
    device tensors: tokens, pred, conf, entropy, renoised."""
    lib = load()
    R = logits.shape[0] if rows is None else rows
    V = logits.shape[-1] if vocab is None else vocab
    stride = logits.stride(0) if row_stride is None else row_stride
    dev = logits.device
    o = outputs if outputs is not None else {
        "tokens": torch.empty(R, dtype=torch.int32, device=dev),
        "pred": torch.empty(R, dtype=torch.int32, device=dev),
        "conf": torch.empty(R, dtype=torch.float32, device=dev),
        "entropy": torch.empty(R, dtype=torch.float32, device=dev),
        "renoised": torch.empty(R, dtype=torch.uint8, device=dev),
    }
    if workspace is None:
        workspace = new_workspace(sample_workspace_bytes(R, V, logits.dtype), dev, stream)
    prm = SampleParams(float(temperature), float(rate), int(seed), int(step), int(row_offset))
    _check(lib.dd_sample_renoise(_ptr(logits), _dtype_code(logits), R, V, stride,
                                 ctypes.byref(prm), _ptr(o["tokens"]), _ptr(o.get("pred")),
                                 _ptr(o["conf"]), _ptr(o.get("entropy")), _ptr(o.get("renoised")),
                                 _ptr(workspace), workspace.numel(), _stream(stream)))
    return o


def sample_renoise_noalloc(logits: torch.Tensor, temperature: float, rate: float, seed: int,
                           step: int, row_offset: int = 0, outputs: Optional[dict] = None,
                           stream=None) -> dict:
    """dd_sample_renoise_noalloc: the sampler step with the library's static
    scratch instead of a workspace (for callers that must not allocate).
    Calls must not overlap on the GPU; see include/dd.h."""
    lib = load()
    R, V = logits.shape[0], logits.shape[-1]
    dev = logits.device
    o = outputs if outputs is not None else {
        "tokens": torch.empty(R, dtype=torch.int32, device=dev),
        "pred": torch.empty(R, dtype=torch.int32, device=dev),
        "conf": torch.empty(R, dtype=torch.float32, device=dev),
        "entropy": torch.empty(R, dtype=torch.float32, device=dev),
        "renoised": torch.empty(R, dtype=torch.uint8, device=dev),
    }
    prm = SampleParams(float(temperature), float(rate), int(seed), int(step), int(row_offset))
    _check(lib.dd_sample_renoise_noalloc(_ptr(logits), _dtype_code(logits), R, V,
                                         logits.stride(0), ctypes.byref(prm), _ptr(o["tokens"]),
                                         _ptr(o.get("pred")), _ptr(o["conf"]),
                                         _ptr(o.get("entropy")), _ptr(o.get("renoised")),
                                         _stream(stream)))
    return o


def init_canvas(rows: int, vocab: int, seed: int, row_offset: int = 0, out=None, device=None,
                stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(rows, dtype=torch.int32, device=device or "cuda")
    _check(load().dd_init_canvas(_ptr(out), rows, vocab, int(seed), int(row_offset),
                                 _stream(stream)))
    return out


def denoise_block_workspace_bytes(desc: AttnDesc, cu_prefix_host, vocab: int) -> int:
    cu = _host_i32(cu_prefix_host)
    return int(load().dd_denoise_block_workspace(ctypes.byref(desc),
                                                 cu.ctypes.data_as(ctypes.c_void_p), vocab))


def denoise_block(q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps,
                  rates: Sequence[float], temperatures: Sequence[float], seed: int, step0: int = 0,
                  cu_prefix_host=None, scale=None, attn_out=None, canvas=None,
                  canvas_history=None, conf_steps=None, keep_history=True, workspace=None,
                  stream=None) -> dict:
    """dd_denoise_block: S steps of attention + sampler/re-noise.

    q_steps [S,B,C,Hq,D], kc/vc_steps [S,B,C,Hkv,D], logits_steps [S,B*C,V].
    Returns dict(attn_out, canvas, canvas_history, conf_steps)."""
    return _block_loop(None, q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps, rates,
                       temperatures, seed, step0, cu_prefix_host, scale, attn_out, canvas,
                       canvas_history, conf_steps, keep_history, workspace, stream)


def denoise_block_fp8(q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, scales_steps,
                      logits_steps, rates: Sequence[float], temperatures: Sequence[float],
                      seed: int, step0: int = 0, cu_prefix_host=None, scale=None, attn_out=None,
                      canvas=None, canvas_history=None, conf_steps=None, keep_history=True,
                      workspace=None, stream=None) -> dict:
    """dd_denoise_block_fp8: as denoise_block with float8_e4m3fn attention
    inputs, scales_steps = one (f_q, f_k, f_v) per step, bf16 logits; the
    attention output is bf16."""
    return _block_loop(scales_steps, q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps,
                       rates, temperatures, seed, step0, cu_prefix_host, scale, attn_out, canvas,
                       canvas_history, conf_steps, keep_history, workspace, stream)


def _block_loop(scales_steps, q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps, rates,
                temperatures, seed, step0, cu_prefix_host, scale, attn_out, canvas,
                canvas_history, conf_steps, keep_history, workspace, stream) -> dict:
    lib = load()
    S = q_steps.shape[0]
    desc = attn_desc(q_steps[0], kc_steps[0], scale)
    cu_h = _host_i32(cu_prefix if cu_prefix_host is None else cu_prefix_host)
    V = logits_steps.shape[-1]
    R = desc.batch * desc.canvas
    dev = q_steps.device
    if attn_out is None:
        attn_out = torch.empty(q_steps.shape, device=dev, dtype=(
            q_steps.dtype if scales_steps is None else torch.bfloat16))
    if canvas is None:
        canvas = torch.empty(R, dtype=torch.int32, device=dev)
    if keep_history and canvas_history is None:
        canvas_history = torch.empty((S, R), dtype=torch.int32, device=dev)
    if keep_history and conf_steps is None:
        conf_steps = torch.empty((S, R), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(denoise_block_workspace_bytes(desc, cu_h, V), dev, stream)
    rates_h = np.ascontiguousarray(np.asarray(rates, dtype=np.float32))
    temps_h = np.ascontiguousarray(np.asarray(temperatures, dtype=np.float32))
    assert rates_h.size >= S and temps_h.size >= S
    head = (ctypes.byref(desc), S, _ptr(q_steps), _ptr(kc_steps), _ptr(vc_steps), _ptr(kp),
            _ptr(vp), _ptr(cu_prefix), cu_h.ctypes.data_as(ctypes.c_void_p))
    tail = (_ptr(attn_out), _ptr(logits_steps), V, rates_h.ctypes.data_as(ctypes.c_void_p),
            temps_h.ctypes.data_as(ctypes.c_void_p), int(seed), int(step0), _ptr(canvas),
            _ptr(canvas_history), _ptr(conf_steps), _ptr(workspace), workspace.numel(),
            _stream(stream))
    if scales_steps is None:
        _check(lib.dd_denoise_block(*head, *tail))
    else:
        assert len(scales_steps) >= S
        f = (Fp8Scales * max(S, 1))(*(Fp8Scales(*(float(x) for x in scales_steps[i]))
                                      for i in range(S)))
        _check(lib.dd_denoise_block_fp8(*head, ctypes.cast(f, ctypes.c_void_p), *tail))
    return {"attn_out": attn_out, "canvas": canvas, "canvas_history": canvas_history,
            "conf_steps": conf_steps}


def soft_embed_workspace_bytes(rows: int, vocab: int, d: int) -> int:
    return int(load().dd_soft_embed_workspace(rows, vocab, d))


def soft_embed(logits: torch.Tensor, temperature: float, emb: torch.Tensor, out=None,
               rows: Optional[int] = None, vocab: Optional[int] = None,
               row_stride: Optional[int] = None, workspace=None, stream=None) -> torch.Tensor:
    """dd_soft_embed: softmax(logits / temperature) @ emb, bf16 [rows, d]."""
    lib = load()
    R = logits.shape[0] if rows is None else rows
    V = logits.shape[-1] if vocab is None else vocab
    stride = logits.stride(0) if row_stride is None else row_stride
    d = emb.shape[-1]
    if out is None:
        out = torch.empty((R, d), dtype=torch.bfloat16, device=logits.device)
    if workspace is None:
        workspace = new_workspace(soft_embed_workspace_bytes(R, V, d), logits.device, stream)
    _check(lib.dd_soft_embed(_ptr(logits), _dtype_code(logits), R, V, stride, float(temperature),
                             _ptr(emb), d, _ptr(out), _ptr(workspace), workspace.numel(),
                             _stream(stream)))
    return out


def ffw(u: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor,
        b2: torch.Tensor, out=None, workspace=None, stream=None) -> torch.Tensor:
    """dd_ffw: the self-conditioning MLP GELU(u w1 + b1) w2 + b2, bf16
    [rows, d] (u [rows, d], w1 [d, h], b1 [h], w2 [h, d], b2 [d], bf16)."""
    lib = load()
    R, d = u.shape
    h = w1.shape[1]
    if out is None:
        out = torch.empty((R, d), dtype=torch.bfloat16, device=u.device)
    if workspace is None:
        workspace = new_workspace(int(lib.dd_ffw_workspace(R, d, h)), u.device, stream)
    _check(lib.dd_ffw(_ptr(u), R, d, h, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(out),
                      _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def self_condition(logits: torch.Tensor, temperature: float, emb: torch.Tensor,
                   w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor, b2: torch.Tensor,
                   out=None, u_out=None, workspace=None, stream=None) -> torch.Tensor:
    """dd_self_condition: z = FFW(softmax(logits / temperature) emb), bf16
    [rows, d]; u_out (optional, bf16 [rows, d]) receives the soft embedding."""
    lib = load()
    R, V = logits.shape
    d = emb.shape[1]
    h = w1.shape[1]
    if out is None:
        out = torch.empty((R, d), dtype=torch.bfloat16, device=logits.device)
    if workspace is None:
        workspace = new_workspace(int(lib.dd_self_condition_workspace(R, V, d, h)),
                                  logits.device, stream)
    _check(lib.dd_self_condition(_ptr(logits), _dtype_code(logits), R, V, logits.stride(0),
                                 float(temperature), _ptr(emb), d, _ptr(w1), _ptr(b1), h,
                                 _ptr(w2), _ptr(b2), _ptr(out), _ptr(u_out), _ptr(workspace),
                                 workspace.numel(), _stream(stream)))
    return out


class BlockGraph:
    """dd_denoise_block captured once (dd_denoise_block_graph_create) and
    replayed with one launch (launch()).  Holds every captured tensor, so the
    buffers outlive the graph; new inputs enter by writing into them
    (`tensors` maps the argument names to those tensors)."""

    _prefix = "dd_denoise_block_graph"

    def __init__(self, handle, tensors: dict, keep: tuple):
        self._h = handle
        self.tensors = tensors
        self._keep = keep

    def launch(self, stream=None):
        if self._h is None:
            raise RuntimeError(f"{type(self).__name__}: destroyed")
        _check(getattr(load(), self._prefix + "_launch")(self._h, _stream(stream)))
        return self.tensors

    def destroy(self):
        if self._h is not None:
            h, self._h = self._h, None
            _check(getattr(load(), self._prefix + "_destroy")(h))

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def denoise_block_graph(q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps,
                        rates: Sequence[float], temperatures: Sequence[float], seed: int,
                        step0: int = 0, cu_prefix_host=None, scale=None, attn_out=None,
                        canvas=None, canvas_history=None, conf_steps=None, keep_history=True,
                        workspace=None) -> BlockGraph:
    """dd_denoise_block_graph_create with the arguments of denoise_block."""
    lib = load()
    S = q_steps.shape[0]
    desc = attn_desc(q_steps[0], kc_steps[0], scale)
    cu_h = _host_i32(cu_prefix if cu_prefix_host is None else cu_prefix_host)
    V = logits_steps.shape[-1]
    R = desc.batch * desc.canvas
    dev = q_steps.device
    if attn_out is None:
        attn_out = torch.empty_like(q_steps)
    if canvas is None:
        canvas = torch.empty(R, dtype=torch.int32, device=dev)
    if keep_history and canvas_history is None:
        canvas_history = torch.empty((S, R), dtype=torch.int32, device=dev)
    if keep_history and conf_steps is None:
        conf_steps = torch.empty((S, R), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = new_workspace(denoise_block_workspace_bytes(desc, cu_h, V), dev)
    rates_h = np.ascontiguousarray(np.asarray(rates, dtype=np.float32))
    temps_h = np.ascontiguousarray(np.asarray(temperatures, dtype=np.float32))
    assert rates_h.size >= S and temps_h.size >= S
    h = ctypes.c_void_p()
    _check(lib.dd_denoise_block_graph_create(
        ctypes.byref(h), ctypes.byref(desc), S, _ptr(q_steps), _ptr(kc_steps), _ptr(vc_steps),
        _ptr(kp), _ptr(vp), _ptr(cu_prefix), cu_h.ctypes.data_as(ctypes.c_void_p),
        _ptr(attn_out), _ptr(logits_steps), V, rates_h.ctypes.data_as(ctypes.c_void_p),
        temps_h.ctypes.data_as(ctypes.c_void_p), int(seed), int(step0), _ptr(canvas),
        _ptr(canvas_history), _ptr(conf_steps), _ptr(workspace), workspace.numel()))
    tensors = {"q_steps": q_steps, "kc_steps": kc_steps, "vc_steps": vc_steps, "kp": kp, "vp": vp,
               "cu_prefix": cu_prefix, "logits_steps": logits_steps, "attn_out": attn_out,
               "canvas": canvas, "canvas_history": canvas_history, "conf_steps": conf_steps,
               "workspace": workspace}
    return BlockGraph(h, tensors, (cu_h, rates_h, temps_h))


def entropy_accept(entropy: torch.Tensor, pred: torch.Tensor, canvas: int, budget: float,
                   seed: int, step: int, vocab: int, row_offset: int = 0, tokens=None,
                   accepted=None, stream=None) -> dict:
    """dd_entropy_accept: the pages' entropy-budget acceptance per canvas."""
    R = entropy.numel()
    if tokens is None:
        tokens = torch.empty(R, dtype=torch.int32, device=entropy.device)
    if accepted is None:
        accepted = torch.empty(R, dtype=torch.uint8, device=entropy.device)
    _check(load().dd_entropy_accept(_ptr(entropy), _ptr(pred), R // canvas, canvas, vocab,
                                    float(budget), int(seed), int(step), int(row_offset),
                                    _ptr(tokens), _ptr(accepted), _stream(stream)))
    return {"tokens": tokens, "accepted": accepted}


def stop_check(entropy: torch.Tensor, pred: torch.Tensor, pred_prev, canvas: int,
               threshold: float, step: int, done: torch.Tensor, halt_step: torch.Tensor,
               stream=None):
    """dd_stop_check: updates done [B] and halt_step [B] in place."""
    _check(load().dd_stop_check(_ptr(entropy), _ptr(pred), _ptr(pred_prev),
                                entropy.numel() // canvas, canvas, float(threshold), int(step),
                                _ptr(done), _ptr(halt_step), _stream(stream)))


def denoise_block_adaptive(q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps,
                           temperatures: Sequence[float], budget: float, stop_entropy: float,
                           seed: int, step0: int = 0, cu_prefix_host=None, scale=None,
                           attn_out=None, canvas=None, keep_history=True, workspace=None,
                           stream=None) -> dict:
    """dd_denoise_block_adaptive: the block loop under the pages' policy.

    Returns dict(canvas, canvas_history [steps_run, R] or None, halt_step [B],
    steps_run)."""
    lib = load()
    S = q_steps.shape[0]
    desc = attn_desc(q_steps[0], kc_steps[0], scale)
    cu_h = _host_i32(cu_prefix if cu_prefix_host is None else cu_prefix_host)
    V = logits_steps.shape[-1]
    R = desc.batch * desc.canvas
    dev = q_steps.device
    if attn_out is None:
        attn_out = torch.empty_like(q_steps)
    if canvas is None:
        canvas = torch.zeros(R, dtype=torch.int32, device=dev)
    history = torch.empty((S, R), dtype=torch.int32, device=dev) if keep_history else None
    halt = torch.empty(desc.batch, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(int(lib.dd_denoise_block_adaptive_workspace(
            ctypes.byref(desc), cu_h.ctypes.data_as(ctypes.c_void_p), V)), dev, stream)
    temps_h = np.ascontiguousarray(np.asarray(temperatures, dtype=np.float32))
    assert temps_h.size >= S
    steps_run = ctypes.c_int(0)
    _check(lib.dd_denoise_block_adaptive(
        ctypes.byref(desc), S, _ptr(q_steps), _ptr(kc_steps), _ptr(vc_steps), _ptr(kp), _ptr(vp),
        _ptr(cu_prefix), cu_h.ctypes.data_as(ctypes.c_void_p), _ptr(attn_out),
        _ptr(logits_steps), V, temps_h.ctypes.data_as(ctypes.c_void_p), float(budget),
        float(stop_entropy), int(seed), int(step0), _ptr(canvas), _ptr(history), _ptr(halt),
        ctypes.byref(steps_run), _ptr(workspace), workspace.numel(), _stream(stream)))
    n = steps_run.value
    return {"canvas": canvas, "canvas_history": None if history is None else history[:n],
            "halt_step": halt, "steps_run": n}


class AdaptiveGraph(BlockGraph):
    """dd_denoise_block_adaptive captured once with the loop on the device
    (dd_denoise_block_adaptive_graph_create); launch() replays it without
    any host synchronisation.  tensors["steps_run"] is a device int32 [1]."""
    _prefix = "dd_denoise_block_adaptive_graph"


def denoise_block_adaptive_graph(q_steps, kc_steps, vc_steps, kp, vp, cu_prefix, logits_steps,
                                 temperatures: Sequence[float], budget: float,
                                 stop_entropy: float, seed: int, step0: int = 0,
                                 cu_prefix_host=None, scale=None, attn_out=None, canvas=None,
                                 keep_history=True, workspace=None) -> AdaptiveGraph:
    """dd_denoise_block_adaptive_graph_create with the arguments of
    denoise_block_adaptive."""
    lib = load()
    S = q_steps.shape[0]
    desc = attn_desc(q_steps[0], kc_steps[0], scale)
    cu_h = _host_i32(cu_prefix if cu_prefix_host is None else cu_prefix_host)
    V = logits_steps.shape[-1]
    R = desc.batch * desc.canvas
    dev = q_steps.device
    if attn_out is None:
        attn_out = torch.empty_like(q_steps)
    if canvas is None:
        canvas = torch.zeros(R, dtype=torch.int32, device=dev)
    history = torch.empty((S, R), dtype=torch.int32, device=dev) if keep_history else None
    halt = torch.empty(desc.batch, dtype=torch.int32, device=dev)
    steps_run = torch.zeros(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(int(lib.dd_denoise_block_adaptive_workspace(
            ctypes.byref(desc), cu_h.ctypes.data_as(ctypes.c_void_p), V)), dev)
    temps_h = np.ascontiguousarray(np.asarray(temperatures, dtype=np.float32))
    assert temps_h.size >= S
    h = ctypes.c_void_p()
    _check(lib.dd_denoise_block_adaptive_graph_create(
        ctypes.byref(h), ctypes.byref(desc), S, _ptr(q_steps), _ptr(kc_steps), _ptr(vc_steps),
        _ptr(kp), _ptr(vp), _ptr(cu_prefix), cu_h.ctypes.data_as(ctypes.c_void_p),
        _ptr(attn_out), _ptr(logits_steps), V, temps_h.ctypes.data_as(ctypes.c_void_p),
        float(budget), float(stop_entropy), int(seed), int(step0), _ptr(canvas), _ptr(history),
        _ptr(halt), _ptr(steps_run), _ptr(workspace), workspace.numel()))
    tensors = {"q_steps": q_steps, "kc_steps": kc_steps, "vc_steps": vc_steps, "kp": kp, "vp": vp,
               "cu_prefix": cu_prefix, "logits_steps": logits_steps, "attn_out": attn_out,
               "canvas": canvas, "canvas_history": history, "halt_step": halt,
               "steps_run": steps_run, "workspace": workspace}
    return AdaptiveGraph(h, tensors, (cu_h, temps_h))


def query_device_error(workspace: torch.Tensor, stream=None):
    _check(load().dd_query_device_error(_ptr(workspace), _stream(stream)))


def set_test_stall_ns(ns: int):
    """dd_set_test_stall_ns: with ns != 0 the tensor-core kernels launched
    afterwards from this thread stall on a barrier nothing completes and
    report DD_ERR_DEVICE_TIMEOUT after ns nanoseconds (0 turns it off)."""
    load().dd_set_test_stall_ns(int(ns))


def launch_count() -> int:
    return int(load().dd_launch_count())


def reset_launch_count():
    load().dd_reset_launch_count()


def status_string(code: int) -> str:
    return load().dd_status_string(code).decode()


def last_error() -> str:
    return load().dd_last_error().decode()
