"""dd_sample_renoise_noalloc: the sampler step for callers that cannot
allocate device memory (code inside another framework's memory pool or
fixed budget, plugin or callback code handed only its buffers, loops that
cannot accept cudaMalloc's device synchronisation).  Instead of a caller
workspace it uses the library's static device scratch.

Checked through the C ABI against dd_sample_renoise (same kernels, so the
outputs must agree to the tolerances of the other sampler tests: token ids
exactly, confidences and entropies within 1e-5), on two calls in a row with
different shapes, so the second call runs on the scratch the first one
left behind.  Collected last on purpose (file name), so that a failure here
cannot hide another test's result.
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


def _noalloc_abi(logits, tau, rate, seed, step, row_offset=0):
    """Direct C-ABI call of dd_sample_renoise_noalloc."""
    lib = dd.load()
    R, V = logits.shape
    o = _outputs(R)
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
