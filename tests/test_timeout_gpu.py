"""The device-timeout path of the tensor-core kernels (attention, soft
embedding, MLP).  With dd_set_test_stall_ns each CTA, once its first MMAs
are in flight, waits on an mbarrier that nothing completes, limited to
100 us.  The call must then report DD_ERR_DEVICE_TIMEOUT through
dd_query_device_error, every CTA must have drained its copies and MMAs and
freed its tensor memory (the next kernels allocate it again on every SM),
and a normal call on the cleared workspace must give the oracle's result.
No fault, trap or unbounded wait is involved: the waits that drain keep
their 1 s limit."""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads
from parity import check_attn

pytestmark = pytest.mark.gpu

DEV = "cuda"
TIMEOUT = 5  # DD_ERR_DEVICE_TIMEOUT


def _expect_timeout(ws):
    with pytest.raises(dd.DDError) as e:
        dd.query_device_error(ws)
    assert e.value.status == TIMEOUT


def _clear(ws):
    dd._check(dd.load().dd_workspace_init(dd._ptr(ws), ws.numel(), dd._stream(None)))


def test_attention_timeout_is_reported_and_the_next_call_is_right():
    w = workloads.scaled(workloads.WORKLOADS["b1_L4096"], prefix_lens=(700,), name="timeout")
    q, kc, vc = (t.to(DEV) for t in workloads.canvas_qkv(w, 0))
    kp, vp, cu = workloads.prefix_kv(w)
    kp, vp, cud = kp.to(DEV), vp.to(DEV), cu.to(DEV)
    desc = dd.attn_desc(q, kc, w.scale)
    ws = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, cu.numpy()), DEV)
    out = torch.zeros_like(q)
    dd.set_test_stall_ns(100_000)
    try:
        dd.canvas_attn(q, kc, vc, kp, vp, cud, cu, scale=w.scale, out=out, workspace=ws)
        _expect_timeout(ws)
    finally:
        dd.set_test_stall_ns(0)
    _clear(ws)
    for _ in range(2):  # every SM allocates tensor memory again
        dd.canvas_attn(q, kc, vc, kp, vp, cud, cu, scale=w.scale, out=out, workspace=ws)
        dd.query_device_error(ws)
    ref, _ = oracle.canvas_attn(q.cpu(), kc.cpu(), vc.cpu(), kp.cpu(), vp.cpu(), cu.numpy(),
                                w.scale, positions=np.array([0, 99, 255], np.int32))
    check_attn(out, ref, torch.bfloat16, positions=np.array([0, 99, 255]))


def test_soft_embed_and_mlp_timeouts_are_reported_and_recover():
    w = workloads.scaled(workloads.WORKLOADS["b1_L4096"], vocab=8192, name="timeout_se")
    lg = workloads.logits(w, 0, device=DEV)
    E = workloads.embedding(w, device=DEV)
    w1, b1, w2, b2 = (t.to(DEV) for t in workloads.ffw_weights(w))
    lib = dd.load()
    ws_se = dd.new_workspace(dd.soft_embed_workspace_bytes(w.rows, w.vocab, E.shape[1]), DEV)
    ws_ff = dd.new_workspace(int(lib.dd_ffw_workspace(w.rows, E.shape[1], w1.shape[1])), DEV)
    u = torch.empty((w.rows, E.shape[1]), dtype=torch.bfloat16, device=DEV)
    z = torch.empty_like(u)
    dd.set_test_stall_ns(100_000)
    try:
        dd.soft_embed(lg, 1.0, E, out=u, workspace=ws_se)
        _expect_timeout(ws_se)
        dd.ffw(u, w1, b1, w2, b2, out=z, workspace=ws_ff)
        _expect_timeout(ws_ff)
    finally:
        dd.set_test_stall_ns(0)
    _clear(ws_se)
    _clear(ws_ff)
    dd.soft_embed(lg, 1.0, E, out=u, workspace=ws_se)
    dd.ffw(u, w1, b1, w2, b2, out=z, workspace=ws_ff)
    dd.query_device_error(ws_se)
    dd.query_device_error(ws_ff)
    ref_u = oracle.soft_embed(lg.cpu(), 1.0, E.cpu())
    got_u = u.float().cpu().numpy()
    assert np.sqrt(((got_u - ref_u) ** 2).mean() / (ref_u ** 2).mean()) <= 8e-3
    ref_z = oracle.ffw(u.cpu(), w1.cpu(), b1.cpu(), w2.cpu(), b2.cpu())
    got_z = z.float().cpu().numpy()
    assert np.sqrt(((got_z - ref_z) ** 2).mean() / (ref_z ** 2).mean()) <= 8e-3
