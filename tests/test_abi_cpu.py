"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/dd.h declares, answers workspace queries, and rejects
invalid arguments before any launch (no CUDA call is reached)."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_discrete_diffusion_dd_b200 as dd
from block_discrete_diffusion_dd_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return dd.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "dd.h")).read()
    return sorted(set(re.findall(r"^DD_API[^(]*?\b(dd_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 12
    assert set(names) == set(dd.EXPORTS)
    for n in names:
        assert getattr(lib, n) is not None
    # and nothing else with the dd_ prefix is exported
    out = os.popen(f"nm -D --defined-only {dd.LIB_PATH}").read()
    exported = sorted(set(re.findall(r" T (dd_\w+)$", out, re.M)))
    assert exported == names


def test_status_strings(lib):
    for code in range(7):
        assert dd.status_string(code)
    assert dd.status_string(99) == "unknown status"


def _desc(B=1, C=256, Hq=16, Hkv=8, D=128, dtype=dd.DD_BF16, scale=None):
    return dd.AttnDesc(B, C, Hq, Hkv, D, scale if scale is not None else D ** -0.5, dtype)


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def test_workspace_queries(lib):
    d = _desc()
    n = dd.canvas_attn_workspace_bytes(d, _cu([4096]))
    assert n > 256
    assert dd.canvas_attn_workspace_bytes(_desc(Hq=6, Hkv=4), _cu([4096])) == 0  # Hq % Hkv
    assert dd.canvas_attn_workspace_bytes(_desc(D=96), _cu([4096])) == 0         # head_dim
    assert dd.canvas_attn_workspace_bytes(_desc(B=2), np.array([0, 5, 3], np.int32)) == 0
    s = dd.sample_workspace_bytes(256, 262144)
    assert s >= 256 + 256 * 32
    assert lib.dd_sample_renoise_workspace(-1, 10, 0) == 0
    assert lib.dd_sample_renoise_workspace(4, 0, 0) == 0
    b = dd.denoise_block_workspace_bytes(d, _cu([4096]), 262144)
    assert b >= max(n, s)


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first


def _sample(lib, rows=4, vocab=16, stride=16, temp=1.0, rate=0.5, dtype=0, tokens=FAKE,
            conf=FAKE, ws=FAKE, ws_bytes=1 << 20, logits=FAKE, row_offset=0):
    p = dd.SampleParams(temp, rate, 0, 0, row_offset)
    return lib.dd_sample_renoise(logits, dtype, rows, vocab, stride, ctypes.byref(p), tokens, None,
                                 conf, None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(rows=-1), 1), (dict(vocab=0), 1), (dict(stride=8), 1), (dict(temp=0.0), 1),
    (dict(temp=float("nan")), 1), (dict(rate=1.5), 1), (dict(rate=-0.1), 1), (dict(dtype=7), 1),
    (dict(tokens=None), 1), (dict(conf=None), 1), (dict(logits=None), 1),
    (dict(ws=None), 3), (dict(ws_bytes=16), 3), (dict(ws=ctypes.c_void_p((1 << 20) + 8)), 3),
    (dict(rows=2, row_offset=0xFFFFFFFF), 1),
])
def test_sampler_rejects_bad_arguments(lib, kw, code):
    assert _sample(lib, **kw) == code
    assert dd.last_error()


def test_sampler_zero_rows_is_a_no_op(lib):
    assert _sample(lib, rows=0, tokens=None, conf=None, logits=None, ws=None) == 0


def _attn(lib, desc, cu, ws_bytes=1 << 30, ptr=FAKE, ws=FAKE, cu_dev=FAKE, kp=FAKE):
    return lib.dd_canvas_attn(ctypes.byref(desc), ptr, ptr, ptr, kp, kp, cu_dev,
                              cu.ctypes.data_as(ctypes.c_void_p), ptr, None, ws, ws_bytes, None)


@pytest.mark.parametrize("desc,cu,code", [
    (_desc(Hq=6, Hkv=4), _cu([16]), 1),
    (_desc(D=96), _cu([16]), 2),
    (_desc(C=0), _cu([16]), 1),
    (_desc(scale=0.0), _cu([16]), 1),
    (_desc(dtype=5), _cu([16]), 1),
    (_desc(B=2), np.array([0, 9, 3], np.int32), 1),
    (_desc(B=2), np.array([1, 9, 30], np.int32), 1),
])
def test_attention_rejects_bad_arguments(lib, desc, cu, code):
    assert _attn(lib, desc, cu) == code
    assert dd.last_error()


def test_attention_rejects_null_and_misaligned(lib):
    d = _desc()
    cu = _cu([16])
    assert _attn(lib, d, cu, ptr=None) == 1
    assert _attn(lib, d, cu, kp=None) == 1                       # prefix rows exist
    assert _attn(lib, d, cu, ptr=ctypes.c_void_p((1 << 20) + 2)) == 1
    assert _attn(lib, d, cu, ws=None) == 3
    assert _attn(lib, d, cu, ws_bytes=300) == 3
    assert _attn(lib, _desc(B=0), cu[:1]) == 0                   # empty batch: no-op


def _attn_fp8(lib, desc, cu, scales=(1.0, 1.0, 1.0), ptr=FAKE, ws=FAKE, ws_bytes=1 << 30):
    f = None if scales is None else ctypes.byref(dd.Fp8Scales(*scales))
    return lib.dd_canvas_attn_fp8(ctypes.byref(desc), ptr, ptr, ptr, ptr, ptr, FAKE,
                                  cu.ctypes.data_as(ctypes.c_void_p), f, ptr, None, ws, ws_bytes,
                                  None)


def test_fp8_attention_rejects_bad_arguments(lib):
    cu = _cu([16])
    e4 = _desc(dtype=dd.DD_E4M3)
    assert _attn(lib, e4, cu) == 1                                  # needs the fp8 entry
    assert "dd_canvas_attn_fp8" in dd.last_error()
    assert _attn_fp8(lib, _desc(), cu) == 1                         # bf16 desc
    assert _attn_fp8(lib, e4, cu, scales=None) == 1
    for bad in ((0.0, 1.0, 1.0), (1.0, -1.0, 1.0), (1.0, 1.0, float("inf")),
                (1.0, float("nan"), 1.0), (1e30, 1e30, 1.0)):
        assert _attn_fp8(lib, e4, cu, scales=bad) == 1, bad
    assert _attn_fp8(lib, _desc(D=64, dtype=dd.DD_E4M3), cu) == 2   # no kernel for D = 64
    assert _attn_fp8(lib, _desc(Hq=12, Hkv=4, dtype=dd.DD_E4M3), cu) == 2  # group 3 !| 128
    assert _attn_fp8(lib, e4, cu, ptr=ctypes.c_void_p((1 << 20) + 4)) == 1
    assert _attn_fp8(lib, e4, cu, ws_bytes=300) == 3
    assert dd.canvas_attn_workspace_bytes(e4, cu) > 0


def _soft(lib, rows=4, vocab=100, stride=104, temp=1.0, d=128, dtype=0, ptr=FAKE, ws=FAKE,
          ws_bytes=1 << 30):
    return lib.dd_soft_embed(ptr, dtype, rows, vocab, stride, temp, ptr, d, ptr, ws, ws_bytes,
                             None)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=1), 2), (dict(dtype=9), 1), (dict(d=96), 2), (dict(d=0), 2), (dict(stride=99), 1),
    (dict(stride=101), 1), (dict(temp=0.0), 1), (dict(temp=float("inf")), 1), (dict(vocab=0), 1),
    (dict(rows=-1), 1), (dict(ptr=None), 1), (dict(ptr=ctypes.c_void_p((1 << 20) + 8)), 1),
    (dict(ws=None), 3), (dict(ws_bytes=512), 3),
])
def test_soft_embed_rejects_bad_arguments(lib, kw, code):
    assert _soft(lib, **kw) == code
    assert dd.last_error()


def test_soft_embed_workspace_and_empty_call(lib):
    assert _soft(lib, rows=0, ptr=None, ws=None) == 0
    assert lib.dd_soft_embed_workspace(256, 262144, 100) == 0
    n = lib.dd_soft_embed_workspace(256, 262144, 2048)
    assert n >= 256 + 256 * 4 + 256 * 2048 * 4   # at least one split of fp32 partials


def _ffw(lib, rows=4, d=64, h=32, ptr=FAKE, w=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return lib.dd_ffw(ptr, rows, d, h, w, w, w, w, ptr, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=8), 1), (dict(h=0), 1), (dict(d=72), 2), (dict(h=40), 2), (dict(rows=-1), 1),
    (dict(ptr=None), 1), (dict(w=None), 1), (dict(w=ctypes.c_void_p((1 << 20) + 4)), 1),
    (dict(ws=None), 3), (dict(ws_bytes=300), 3),
])
def test_ffw_rejects_bad_arguments(lib, kw, code):
    assert _ffw(lib, **kw) == code
    assert dd.last_error()


def test_ffw_workspace_and_empty_call(lib):
    assert _ffw(lib, rows=0, ptr=None, w=None, ws=None) == 0
    assert lib.dd_ffw_workspace(256, 2048, 1904) >= 256 + 256 * 1904 * 2
    assert lib.dd_ffw_workspace(256, 2048, 1900) == 0
    n = lib.dd_self_condition_workspace(256, 262144, 2048, 1904)
    assert n >= lib.dd_soft_embed_workspace(256, 262144, 2048) + 256 * (2048 + 1904) * 2
    assert lib.dd_self_condition_workspace(256, 262144, 2000, 1904) == 0


def _selfcond(lib, rows=4, vocab=100, stride=104, d=128, h=32, dtype=0, ptr=FAKE, w=FAKE,
              u_out=None, ws=FAKE, ws_bytes=1 << 30):
    return lib.dd_self_condition(ptr, dtype, rows, vocab, stride, 1.0, ptr, d, w, w, h, w, w, ptr,
                                 u_out, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=1), 2), (dict(d=96), 2), (dict(h=24), 2), (dict(stride=99), 1), (dict(w=None), 1),
    (dict(u_out=ctypes.c_void_p((1 << 20) + 2)), 1), (dict(ws=None), 3), (dict(ws_bytes=512), 3),
])
def test_self_condition_rejects_bad_arguments(lib, kw, code):
    assert _selfcond(lib, **kw) == code
    assert dd.last_error()


def test_block_graph_rejects_bad_handles(lib):
    d = _desc()
    cu = _cu([16])
    r = np.zeros(1, np.float32)
    args = [ctypes.byref(d), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
            cu.ctypes.data_as(ctypes.c_void_p), FAKE, FAKE, 1024,
            r.ctypes.data_as(ctypes.c_void_p), r.ctypes.data_as(ctypes.c_void_p), 0, 0, FAKE,
            None, None, FAKE, 16]
    assert lib.dd_denoise_block_graph_create(None, *args) == 1       # no handle slot
    assert lib.dd_denoise_block_graph_launch(None, None) == 1
    assert lib.dd_denoise_block_graph_destroy(None) == 0


def test_block_rejects_bad_arguments(lib):
    d = _desc()
    cu = _cu([16])
    r = np.zeros(1, np.float32)
    args = [ctypes.byref(d), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
            cu.ctypes.data_as(ctypes.c_void_p), FAKE, FAKE, 1024,
            r.ctypes.data_as(ctypes.c_void_p), r.ctypes.data_as(ctypes.c_void_p), 0, 0, FAKE,
            None, None, FAKE, 16, None]
    assert lib.dd_denoise_block(*args) == 3                      # workspace too small
    bad = list(args)
    bad[1] = -1
    assert lib.dd_denoise_block(*bad) == 1
    bad = list(args)
    bad[12] = None
    assert lib.dd_denoise_block(*bad) == 1
    bad = list(args)
    bad[16] = None
    assert lib.dd_denoise_block(*bad) == 1


def test_block_fp8_rejects_bad_arguments(lib):
    e4 = _desc(dtype=dd.DD_E4M3)
    cu = _cu([16])
    cuh = cu.ctypes.data_as(ctypes.c_void_p)
    r = np.zeros(2, np.float32)
    rp = r.ctypes.data_as(ctypes.c_void_p)
    good = (dd.Fp8Scales * 2)(dd.Fp8Scales(1.0, 1.0, 1.0), dd.Fp8Scales(0.5, 2.0, 1.0))
    ws = lib.dd_denoise_block_workspace(ctypes.byref(e4), cuh, 1024)
    assert ws > 0                                               # E4M3 geometry is queried

    def call(desc=e4, scales=ctypes.cast(good, ctypes.c_void_p), ws_bytes=ws, steps=2):
        return lib.dd_denoise_block_fp8(ctypes.byref(desc), steps, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, cuh, scales, FAKE, FAKE, 1024, rp, rp, 0, 0, FAKE,
                                        None, None, FAKE, ws_bytes, None)

    assert call(ws_bytes=16) == 3                                # workspace too small
    assert call(desc=_desc()) == 1                               # bf16 desc
    assert "DD_E4M3" in dd.last_error()
    assert call(scales=None) == 1
    for bad in ((0.0, 1.0, 1.0), (1.0, float("nan"), 1.0), (1e30, 1e30, 1.0)):
        sc = (dd.Fp8Scales * 2)(dd.Fp8Scales(1.0, 1.0, 1.0), dd.Fp8Scales(*bad))
        assert call(scales=ctypes.cast(sc, ctypes.c_void_p)) == 1, bad
        assert "step 1" in dd.last_error()
    assert call(scales=None, steps=0, ws_bytes=16) == 3          # steps 0: factors unused
    args = [ctypes.byref(e4), 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, cuh, FAKE, FAKE, 1024, rp,
            rp, 0, 0, FAKE, None, None, FAKE, ws, None]
    assert lib.dd_denoise_block(*args) == 1                      # E4M3 needs the fp8 entry
    assert "dd_denoise_block_fp8" in dd.last_error()


def test_adaptive_graph_rejects_bad_arguments(lib):
    d = _desc()
    cu = _cu([16])
    t = np.full(2, 0.8, np.float32)
    h = ctypes.c_void_p(123)

    def create(out=ctypes.byref(h), steps_run=FAKE, ws_bytes=16, canvas=FAKE, temps=True):
        return lib.dd_denoise_block_adaptive_graph_create(
            out, ctypes.byref(d), 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
            cu.ctypes.data_as(ctypes.c_void_p), FAKE, FAKE, 1024,
            t.ctypes.data_as(ctypes.c_void_p) if temps else None, 0.1, 0.005, 0, 0, canvas,
            None, FAKE, steps_run, FAKE, ws_bytes)

    assert create(out=None) == 1
    assert create() == 3 and h.value is None                 # workspace too small; no handle
    assert create(steps_run=None) == 1
    assert create(canvas=None) == 1
    assert create(temps=False) == 1
    assert lib.dd_denoise_block_adaptive_graph_launch(None, None) == 1
    assert lib.dd_denoise_block_adaptive_graph_destroy(None) == 0


def test_init_canvas_rejects_bad_arguments(lib):
    assert lib.dd_init_canvas(None, 4, 10, 0, 0, None) == 1
    assert lib.dd_init_canvas(FAKE, 4, 0, 0, 0, None) == 1
    assert lib.dd_init_canvas(None, 0, 10, 0, 0, None) == 0


def test_policy_entries_reject_bad_arguments(lib):
    acc = lib.dd_entropy_accept
    assert acc(FAKE, FAKE, 2, 2000, 16, 0.1, 0, 0, 0, FAKE, None, None) == 1      # canvas > 1024
    assert acc(FAKE, FAKE, 2, 0, 16, 0.1, 0, 0, 0, FAKE, None, None) == 1
    assert acc(FAKE, FAKE, 2, 8, 0, 0.1, 0, 0, 0, FAKE, None, None) == 1          # vocab
    assert acc(FAKE, FAKE, 2, 8, 16, float("nan"), 0, 0, 0, FAKE, None, None) == 1
    assert acc(None, FAKE, 2, 8, 16, 0.1, 0, 0, 0, FAKE, None, None) == 1
    assert acc(FAKE, FAKE, 2, 8, 16, 0.1, 0, 0, 0, None, None, None) == 1
    assert acc(FAKE, FAKE, 1, 8, 16, 0.1, 0, 0, 0xFFFFFFFC, FAKE, None, None) == 1  # row_offset
    assert acc(None, None, 0, 8, 16, 0.1, 0, 0, 0, None, None, None) == 0         # empty: no-op
    stop = lib.dd_stop_check
    assert stop(FAKE, FAKE, None, 2, 8, 0.005, 0, None, FAKE, None) == 1
    assert stop(FAKE, FAKE, None, 2, 8, 0.005, 0, FAKE, None, None) == 1
    assert stop(FAKE, FAKE, None, -1, 8, 0.005, 0, FAKE, FAKE, None) == 1
    assert stop(None, None, None, 0, 8, 0.005, 0, None, None, None) == 0
    d = _desc()
    cu = _cu([16])
    wa = lib.dd_denoise_block_adaptive_workspace(ctypes.byref(d),
                                                cu.ctypes.data_as(ctypes.c_void_p), 1024)
    wb = lib.dd_denoise_block_workspace(ctypes.byref(d), cu.ctypes.data_as(ctypes.c_void_p), 1024)
    assert wa > wb > 0
    t = np.full(4, 0.8, np.float32)
    n = ctypes.c_int(-5)
    args = [ctypes.byref(d), 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
            cu.ctypes.data_as(ctypes.c_void_p), FAKE, FAKE, 1024,
            t.ctypes.data_as(ctypes.c_void_p), 0.1, 0.005, 0, 0, FAKE, None, FAKE,
            ctypes.byref(n), FAKE, 16, None]
    ad = lib.dd_denoise_block_adaptive
    assert ad(*args) == 3                                         # workspace too small
    for i, v in [(1, -1), (12, None), (17, None), (19, None), (20, None), (13, float("nan"))]:
        bad = list(args)
        bad[i] = v
        assert ad(*bad) == 1, i
    big = _desc(C=2048)
    bad = list(args)
    bad[0] = ctypes.byref(big)
    bad[21] = FAKE
    bad[22] = 1 << 40
    assert ad(*bad) == 2                                          # canvas > 1024
