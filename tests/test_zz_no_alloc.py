"""dd_sample_renoise_noalloc: the sampler step for callers that cannot
allocate device memory (code inside another framework's memory pool or
fixed budget, plugin or callback code handed only its buffers, loops that
cannot accept cudaMalloc's device synchronisation).  Instead of a caller
workspace it uses the library's static device scratch.

Checked through the C ABI against dd_sample_renoise (same kernels, so the
outputs must agree to the tolerances of the other sampler tests: token ids
exactly, confidences and entropies within 1e-5), on two calls in a row with
different shapes, so the second call runs on the scratch the first one
left behind; that a call allocates no device memory (the free memory the
driver reports is the same before and after it); the size limit at its
edge (1927 rows of 262144 entries pass, 1928 are rejected); and correct
results after calls that were rejected.  Collected last on purpose (file
name), so that a failure here cannot hide another test's result.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_discrete_diffusion_dd_b200 as dd
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _outputs(R):
    return {"tokens": torch.full((R,), -1, dtype=torch.int32, device=DEV),
            "pred": torch.full((R,), -1, dtype=torch.int32, device=DEV),
            "conf": torch.full((R,), float("nan"), dtype=torch.float32, device=DEV),
            "entropy": torch.full((R,), float("nan"), dtype=torch.float32, device=DEV),
            "renoised": torch.full((R,), 7, dtype=torch.uint8, device=DEV)}


def _noalloc_abi(logits, tau, rate, seed, step, row_offset=0, o=None):
    """Direct C-ABI call of dd_sample_renoise_noalloc."""
    lib = dd.load()
    R, V = logits.shape
    o = _outputs(R) if o is None else o
    prm = dd.SampleParams(tau, rate, seed, step, row_offset)
    code = dd.DD_BF16 if logits.dtype == torch.bfloat16 else dd.DD_F32
    st = lib.dd_sample_renoise_noalloc(
        ctypes.c_void_p(logits.data_ptr()), code, R, V, logits.stride(0), ctypes.byref(prm),
        ctypes.c_void_p(o["tokens"].data_ptr()), ctypes.c_void_p(o["pred"].data_ptr()),
        ctypes.c_void_p(o["conf"].data_ptr()), ctypes.c_void_p(o["entropy"].data_ptr()),
        ctypes.c_void_p(o["renoised"].data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, dd.last_error()
    torch.cuda.synchronize()
    return o


def _compare(a, b):
    for k in ("tokens", "pred", "renoised"):
        assert torch.equal(a[k], b[k]), k
    for k in ("conf", "entropy"):
        x, y = a[k].double().cpu().numpy(), b[k].double().cpu().numpy()
        np.testing.assert_allclose(x, y, rtol=1e-5, atol=1e-5 * np.abs(y).max())


def test_noalloc_matches_workspace_entry_point_twice():
    w = workloads.WORKLOADS["b1_L4096"]
    big = workloads.logits(w, 0, device=DEV)                       # 256 x 262144 bf16
    tiny_w = workloads.WORKLOADS["tiny_fp32"]
    small = workloads.logits(tiny_w, 0).to(DEV)                    # 256 x 1024 fp32
    calls = [(big, 1.0, 0.3, 0, 0, 0), (small, 0.7, 0.5, 5, 3, 77)]
    for logits, tau, rate, seed, step, off in calls:
        got = _noalloc_abi(logits, tau, rate, seed, step, off)
        ref = dd.sample_renoise(logits, tau, rate, seed, step, off, outputs=_outputs(logits.shape[0]))
        torch.cuda.synchronize()
        _compare(got, ref)
    # and once more on the first shape, after the second call left its records
    got = _noalloc_abi(big, 1.0, 0.3, 0, 0, 0)
    ref = dd.sample_renoise(big, 1.0, 0.3, 0, 0, 0, outputs=_outputs(big.shape[0]))
    torch.cuda.synchronize()
    _compare(got, ref)


def test_noalloc_rejects_calls_beyond_its_scratch():
    lib = dd.load()
    prm = dd.SampleParams(1.0, 0.5, 0, 0, 0)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    st = lib.dd_sample_renoise_noalloc(fake, dd.DD_BF16, 57337, 262144, 262144, ctypes.byref(prm),
                                       fake, None, fake, None, None, None)
    assert st == 2  # DD_ERR_UNSUPPORTED
    assert "static scratch" in dd.last_error()


def test_noalloc_allocates_no_device_memory():
    w = workloads.WORKLOADS["b1_L4096"]
    lg = workloads.logits(w, 0, device=DEV)
    o = _outputs(lg.shape[0])
    _noalloc_abi(lg, 1.0, 0.3, 0, 0, 0, o)           # first call: address look-up, module load
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for step in range(3):
        _noalloc_abi(lg, 1.0, 0.3, 0, step, 0, o)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"


def test_noalloc_size_limit_at_its_edge_and_after_rejected_calls():
    """1927 rows of 262144 bf16 entries fit the 4 MiB scratch and match
    dd_sample_renoise; 1928 do not.  Rejected calls (too large, NULL
    params, a bad temperature) queue nothing, and the next call is right."""
    lib = dd.load()
    V = 262144
    g = torch.Generator(device=DEV).manual_seed(7)
    lg = (torch.randn((1928, V), generator=g, device=DEV) * 3.0).to(torch.bfloat16)
    prm = dd.SampleParams(1.0, 0.25, 3, 1, 0)
    o = _outputs(1928)
    args = lambda rows, p: (ctypes.c_void_p(lg.data_ptr()), dd.DD_BF16, rows, V, V,
                            p, ctypes.c_void_p(o["tokens"].data_ptr()), None,
                            ctypes.c_void_p(o["conf"].data_ptr()), None, None, None)
    assert lib.dd_sample_renoise_noalloc(*args(1928, ctypes.byref(prm))) == 2
    assert "static scratch" in dd.last_error()
    assert lib.dd_sample_renoise_noalloc(*args(1927, None)) == 1         # params NULL
    assert lib.dd_sample_renoise_noalloc(*args(0, None)) == 1            # checked at rows 0 too
    bad = dd.SampleParams(0.0, 0.25, 3, 1, 0)
    assert lib.dd_sample_renoise_noalloc(*args(1927, ctypes.byref(bad))) == 1
    torch.cuda.synchronize()
    assert (o["tokens"] == -1).all()                                     # nothing ran
    got = _noalloc_abi(lg[:1927], 1.0, 0.25, 3, 1, 0)
    ref = dd.sample_renoise(lg[:1927], 1.0, 0.25, 3, 1, 0, outputs=_outputs(1927))
    torch.cuda.synchronize()
    _compare(got, ref)
