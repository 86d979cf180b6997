"""GPU parity of dd_canvas_attn against the float64 oracle.

bf16 inputs with head_dim 128 run on the tcgen05 tensor-core kernel; fp32
inputs and the other geometries run on the CUDA-core kernel.  Sizes span
several 128-key and 128-row tiles with ragged tails (partial prefix tiles,
zero-length prefixes, canvases that are not a multiple of 128); the full
workloads run in their real launch configuration and are checked on sampled
canvas positions.
"""
import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import oracle
import workloads
from parity import check_attn

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _problem(B, C, Hq, Hkv, D, lens, dtype=torch.bfloat16, seed=0, q_gain=1.0, device="cpu"):
    g = torch.Generator(device=device).manual_seed(seed)

    def r(*shape, gain=1.0):
        return (torch.randn(shape, generator=g, device=device) * gain).to(dtype)

    q = r(B, C, Hq, D, gain=q_gain)
    kc, vc = r(B, C, Hkv, D), r(B, C, Hkv, D)
    n = int(sum(lens))
    kp, vp = r(max(n, 0), Hkv, D), r(max(n, 0), Hkv, D)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    return q, kc, vc, kp, vp, cu


def _run(q, kc, vc, kp, vp, cu, scale=None, want_lse=True):
    desc = dd.attn_desc(q, kc, scale)
    ws = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, cu))
    out, lse = dd.canvas_attn(q.to(DEV), kc.to(DEV), vc.to(DEV), kp.to(DEV), vp.to(DEV),
                              cu.to(DEV), cu, scale=scale, want_lse=want_lse, workspace=ws)
    dd.query_device_error(ws)  # synchronises; raises on a latched device error
    return out, lse


def test_tiny_fp32_workload():
    w = workloads.WORKLOADS["tiny_fp32"]
    q, kc, vc = workloads.canvas_qkv(w, 0)
    kp, vp, cu = workloads.prefix_kv(w)
    out, lse = _run(q, kc, vc, kp, vp, cu, w.scale)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), w.scale)
    st = check_attn(out, ref, torch.float32)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=1e-5)
    print("tiny_fp32", st)


@pytest.mark.parametrize("lens,q_gain", [((0, 100, 300), 1.0), ((129, 1, 640), 4.0),
                                         ((4096,), 1.0)])
def test_tensor_core_ragged(lens, q_gain):
    B = len(lens)
    q, kc, vc, kp, vp, cu = _problem(B, 256, 16, 8, 128, lens, seed=len(lens), q_gain=q_gain)
    out, lse = _run(q, kc, vc, kp, vp, cu)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5)
    st = check_attn(out, ref, torch.bfloat16)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)
    print(lens, q_gain, st)


@pytest.mark.parametrize("C,Hq,Hkv,lens", [
    (256, 16, 8, (1536,)),     # 7 splits: the merge shape for up to 8 splits
    (256, 16, 8, (4096,)),     # 9 splits: up to 12
    (256, 8, 4, (1408,)),      # 13 splits: up to 16
    (128, 2, 1, (16384,)),     # one unit per split, about 129 splits: the looped merge
])
def test_tensor_core_split_counts(C, Hq, Hkv, lens):
    q, kc, vc, kp, vp, cu = _problem(len(lens), C, Hq, Hkv, 128, lens, seed=C + Hq)
    out, lse = _run(q, kc, vc, kp, vp, cu)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5)
    check_attn(out, ref, torch.bfloat16)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)


@pytest.mark.parametrize("v_gain", [1e5, 1e-6])
def test_tensor_core_value_range(v_gain):
    # split partials are stored as fp16 scaled per row by a power of two: V
    # far above fp16's range (65504) and far below its normal range must
    # come through with the relative accuracy of unit-scale V
    q, kc, vc, kp, vp, cu = _problem(2, 256, 16, 8, 128, (300, 1000), seed=11)
    vc = (vc.float() * v_gain).to(torch.bfloat16)
    vp = (vp.float() * v_gain).to(torch.bfloat16)
    out, lse = _run(q, kc, vc, kp, vp, cu)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5)
    check_attn(out, ref, torch.bfloat16, max_abs=2e-2 * v_gain)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)


def test_tensor_core_wide_batch():
    # more batch rows than the host's per-row plan holds: the kernels then
    # derive one split length for every row themselves
    lens = tuple(int(x) for x in np.random.default_rng(7).integers(0, 400, 130))
    q, kc, vc, kp, vp, cu = _problem(130, 16, 2, 1, 128, lens, seed=130)
    out, lse = _run(q, kc, vc, kp, vp, cu)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5)
    check_attn(out, ref, torch.bfloat16)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (16, 2), (32, 4)])
def test_tensor_core_head_groupings(Hq, Hkv):
    q, kc, vc, kp, vp, cu = _problem(2, 256, Hq, Hkv, 128, (200, 77), seed=Hq + Hkv)
    out, _ = _run(q, kc, vc, kp, vp, cu)
    ref, _ = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5)
    check_attn(out, ref, torch.bfloat16)


@pytest.mark.parametrize("C", [200, 64, 1])
def test_tensor_core_ragged_canvas(C):
    q, kc, vc, kp, vp, cu = _problem(2, C, 16, 8, 128, (150, 0), seed=C)
    out, _ = _run(q, kc, vc, kp, vp, cu)
    ref, _ = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), 128 ** -0.5)
    check_attn(out, ref, torch.bfloat16)


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 64), (torch.float32, 128),
                                     (torch.float32, 64)])
def test_cuda_core_path(dtype, D):
    q, kc, vc, kp, vp, cu = _problem(2, 96, 4, 2, D, (33, 0), dtype=dtype, seed=D)
    out, lse = _run(q, kc, vc, kp, vp, cu)
    ref, ref_lse = oracle.canvas_attn(q, kc, vc, kp, vp, cu.numpy(), D ** -0.5)
    check_attn(out, ref, dtype)


def test_canvas_permutation_equivariance_on_gpu():
    q, kc, vc, kp, vp, cu = _problem(1, 256, 16, 8, 128, (384,), seed=3, q_gain=3.0)
    out, _ = _run(q, kc, vc, kp, vp, cu)
    perm = torch.randperm(256, generator=torch.Generator().manual_seed(2))
    out_p, _ = _run(q[:, perm].contiguous(), kc[:, perm].contiguous(), vc[:, perm].contiguous(),
                    kp, vp, cu)
    diff = (out_p.float() - out[:, perm.to(DEV)].float()).abs().max().item()
    assert diff <= 2e-2


def _positions(C, n=12, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, 1, C - 1], rng.integers(0, C, n)])).astype(np.int32)


@pytest.mark.parametrize("name", ["b1_L4096", "long_L65536", "ragged_b8"])
def test_full_workloads_sampled(name):
    w = workloads.WORKLOADS[name]
    q, kc, vc = workloads.canvas_qkv(w, 0, device=DEV)
    kp, vp, cu = workloads.prefix_kv(w, device=DEV)
    out, lse = dd.canvas_attn(q, kc, vc, kp, vp, cu.to(DEV), cu, scale=w.scale, want_lse=True)
    torch.cuda.synchronize()
    pos = _positions(w.canvas, 6 if name == "long_L65536" else 12)
    ref, ref_lse = oracle.canvas_attn(q.cpu(), kc.cpu(), vc.cpu(), kp.cpu(), vp.cpu(),
                                      cu.numpy(), w.scale, positions=pos)
    st = check_attn(out, ref, torch.bfloat16, positions=pos)
    np.testing.assert_allclose(lse.cpu().numpy()[:, :, pos], ref_lse[:, :, pos], atol=2e-2)
    print(name, st)


def test_multi_round_merge_repeats_and_replays():
    # The ragged batch takes more than one round of the SMs (240 CTAs), so
    # its split merge polls per-group counters in the workspace that every
    # call must leave cleared: repeated calls on one workspace, and replays
    # of one captured call, give the same bits.
    w = workloads.WORKLOADS["ragged_b8"]
    q, kc, vc = workloads.canvas_qkv(w, 0, device=DEV)
    kp, vp, cu = workloads.prefix_kv(w, device=DEV)
    cud = cu.to(DEV)
    desc = dd.attn_desc(q, kc, w.scale)
    ws = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, cu.numpy()))
    out = torch.empty_like(q)

    def call():
        dd.canvas_attn(q, kc, vc, kp, vp, cud, cu, scale=w.scale, out=out, workspace=ws)

    outs = []
    for _ in range(3):
        call()
        outs.append(out.clone())
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            call()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        outs.append(out.clone())
    dd.query_device_error(ws)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_no_device_error_latched():
    q, kc, vc, kp, vp, cu = _problem(1, 256, 16, 8, 128, (1000,), seed=4)
    desc = dd.attn_desc(q, kc)
    ws = dd.new_workspace(dd.canvas_attn_workspace_bytes(desc, cu))
    dd.canvas_attn(q.to(DEV), kc.to(DEV), vc.to(DEV), kp.to(DEV), vp.to(DEV), cu.to(DEV), cu,
                   workspace=ws)
    dd.query_device_error(ws)  # raises on a latched timeout / bounds error
