"""The no-allocation layer call (oq_qlinear_noalloc) against the ordinary one.

Some callers may not allocate device memory while they run -- a serving
process that reserved all device memory at start-up and forbids
cudaMalloc/cudaFree on its request path.  For them the library offers a
variant of oq_qlinear that takes no workspace and allocates nothing: the
packed activation codes go to a fixed per-device scratch array inside the
library.  These tests call it through the C ABI twice in a row and check
each result against oq_qlinear, which runs the same kernels on a torch
workspace.  The file is collected last so that a failure here cannot hide
the rest of the suite; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from rotation_bit_quantization_rpbh_b200 import binding as B

from parity import GEMM_TOL, rel_frob

pytestmark = pytest.mark.gpu


def _layer(dev, M, d, N, h, bw, ba, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16).to(dev)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16).to(dev)
    plan = B.rpbh_plan(d, h, seed)
    cb_a, cb_w = B.codebook(d, ba), B.codebook(d, bw)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W)
    return plan, cb_a, cb_w, x, w_idx, w_r


@pytest.mark.parametrize("M,d,N,h,bw,ba", [(300, 512, 520, 128, 4, 4), (4096, 3072, 768, 128, 4, 4),
                                           (1000, 1536, 256, 128, 4, 6)])
def test_noalloc_matches_the_allocating_call_twice(cuda_device, M, d, N, h, bw, ba):
    plan, cb_a, cb_w, x, w_idx, w_r = _layer(cuda_device, M, d, N, h, bw, ba, 31)
    ref = B.qlinear(plan, cb_a, cb_w, x, w_idx, w_r)  # also puts the codebook tables on the device
    ref64 = ref.float().cpu().numpy().astype(np.float64)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        B.qlinear_noalloc(plan, cb_a, cb_w, x, w_idx, w_r, y)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got))
        assert rel_frob(got, ref64) <= GEMM_TOL
        assert torch.equal(y, ref)  # the same kernels on the same codes
    assert B.device_status() == 0


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_device):
    plan, cb_a, cb_w, x, w_idx, w_r = _layer(cuda_device, 64, 4096, 256, 128, 4, 4, 32)
    B.qlinear(plan, cb_a, cb_w, x, w_idx, w_r)
    M_big = B.NOALLOC_SCRATCH_BYTES // (4096 // 2) + 1024  # more packed rows than the scratch holds
    assert B.qlinear_workspace(M_big, 4096, 4) > B.NOALLOC_SCRATCH_BYTES
    L = B.lib()
    st = L.oq_qlinear_noalloc(plan.handle, cb_a.handle, cb_w.handle, ctypes.c_void_p(x.data_ptr()), B.OQ_BF16, M_big,
                              ctypes.c_void_p(w_idx.data_ptr()), ctypes.c_void_p(w_r.data_ptr()), 256, None,
                              ctypes.c_void_p(x.data_ptr()), None)
    assert st == 8  # OQ_ERR_TOO_LARGE, before any kernel runs


def test_noalloc_needs_the_codebook_on_the_device_first(cuda_device):
    d = 256
    plan = B.rpbh_plan(d, 64, 33)
    cb_a, cb_w = B.codebook(d, 4), B.codebook(d, 4)  # fresh: no device tables yet
    x = torch.randn(8, d, device=cuda_device).to(torch.bfloat16)
    w_idx = torch.zeros((16, d // 2), dtype=torch.uint8, device=cuda_device)
    w_r = torch.ones(16, dtype=torch.bfloat16, device=cuda_device)
    y = torch.empty((8, 16), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(B.OQError) as e:
        B.qlinear_noalloc(plan, cb_a, cb_w, x, w_idx, w_r, y)
    assert e.value.status == 1


def test_noalloc_reports_too_large_for_eight_bit_values_before_any_work(cuda_device):
    """8-bit activations have no codes schedule (no in-kernel 8-bit decoder),
    so when their values do not fit the scratch the call must return
    OQ_ERR_TOO_LARGE up front -- not quantise into the scratch and then find
    that the product cannot run -- even though the 8-bit codes would fit."""
    d, N, M = 4096, 256, 20000
    plan = B.rpbh_plan(d, 128, 34)
    cb_a, cb_w = B.codebook(d, 8), B.codebook(d, 4)
    cb_a.upload()  # the call itself allocates nothing
    assert B.qlinear_workspace_values(M, d) > B.NOALLOC_SCRATCH_BYTES
    assert B.qlinear_workspace(M, d, 8) <= B.NOALLOC_SCRATCH_BYTES
    x = torch.zeros((M, d), dtype=torch.bfloat16, device=cuda_device)
    w_idx = torch.zeros((N, d // 2), dtype=torch.uint8, device=cuda_device)
    w_r = torch.ones(N, dtype=torch.bfloat16, device=cuda_device)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device=cuda_device)
    L = B.lib()
    st = L.oq_qlinear_noalloc(plan.handle, cb_a.handle, cb_w.handle, ctypes.c_void_p(x.data_ptr()), B.OQ_BF16, M,
                              ctypes.c_void_p(w_idx.data_ptr()), ctypes.c_void_p(w_r.data_ptr()), N, None,
                              ctypes.c_void_p(y.data_ptr()), None)
    torch.cuda.synchronize()
    assert st == 8  # OQ_ERR_TOO_LARGE
    assert B.device_status() == 0
    assert bool((y == 7.0).all())  # nothing was written
