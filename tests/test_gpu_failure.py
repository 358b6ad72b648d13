"""Failure detection on the GPU without a GPU fault.

Failures are made on the host through the library's test hooks:
- an allocation that reports failure must surface as OQ_ERR_OOM and leave
  no partial state behind;
- a launch that issues none of its input copies must end its bounded waits,
  record OQ_ERR_TIMEOUT for ``device_status()`` and leave the context usable
  for the next call, whose results are unchanged.
Each starved launch waits out its limit (about one second)."""
import pytest
import torch

from rotation_bit_quantization_rpbh_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer(cuda_device):
    d, h = 512, 64
    plan = B.rpbh_plan(d, h, 5)
    cb4, cb2 = B.codebook(d, 4), B.codebook(d, 2)
    g = torch.Generator().manual_seed(11)
    x = torch.randn(300, d, generator=g).to(torch.bfloat16).to(cuda_device)
    W = torch.randn(320, d, generator=g).to(torch.bfloat16).to(cuda_device)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    idx, s = B.quantize_acts(plan, cb4, x)
    y = B.qgemm(cb4, cb2, idx, s, w_idx, w_r)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    return dict(plan=plan, cb4=cb4, cb2=cb2, x=x, W=W, w_idx=w_idx, w_r=w_r, idx=idx, s=s, y=y, d=d, h=h)


def _reset_hooks():
    B.debug_starve(0)
    B.debug_fail_allocations(0)


def test_plan_allocation_failure_reports_oom_and_recovers(layer):
    d, h = layer["d"], layer["h"]
    B.debug_fail_allocations(1)
    try:
        with pytest.raises(B.OQError) as e:
            B.rpbh_plan(d, h, 99)
        assert e.value.status == 6  # OQ_ERR_OOM
    finally:
        B.debug_fail_allocations(0)
    plan = B.rpbh_plan(d, h, 99)  # the failure was consumed: the next plan is whole
    idx_a, s_a = B.quantize_acts(plan, layer["cb4"], layer["x"])
    idx_b, s_b = B.quantize_acts(B.rpbh_plan(d, h, 99), layer["cb4"], layer["x"])
    assert torch.equal(idx_a, idx_b) and torch.equal(s_a, s_b)


def test_codebook_upload_failure_reports_oom_and_recovers(layer):
    plan, x = layer["plan"], layer["x"]
    cb = B.codebook(layer["d"], 4)  # a new handle: its table is uploaded on first use
    B.debug_fail_allocations(1)
    try:
        with pytest.raises(B.OQError) as e:
            B.quantize_acts(plan, cb, x)
        assert e.value.status == 6
    finally:
        B.debug_fail_allocations(0)
    idx, s = B.quantize_acts(plan, cb, x)  # the upload is retried, not left half done
    assert torch.equal(idx, layer["idx"]) and torch.equal(s, layer["s"])
    assert B.device_status() == 0


def test_starved_activation_quantizer_times_out_and_context_survives(layer):
    plan, cb4, x = layer["plan"], layer["cb4"], layer["x"]
    B.debug_starve(B.OQ_STARVE_RPBH)
    try:
        B.quantize_acts(plan, cb4, x)  # the launch itself is accepted
        assert B.device_status(clear=True) == 5  # OQ_ERR_TIMEOUT
    finally:
        _reset_hooks()
    assert B.device_status() == 0  # cleared
    idx, s = B.quantize_acts(plan, cb4, x)  # the starve was consumed by one launch
    assert torch.equal(idx, layer["idx"]) and torch.equal(s, layer["s"])
    assert B.device_status() == 0


def test_starved_weight_quantizer_times_out_and_context_survives(layer):
    plan, cb2, W = layer["plan"], layer["cb2"], layer["W"]
    B.debug_starve(B.OQ_STARVE_RPBH)
    try:
        B.quantize_weights(plan, cb2, W)
        assert B.device_status(clear=True) == 5
    finally:
        _reset_hooks()
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    assert torch.equal(w_idx, layer["w_idx"]) and torch.equal(w_r, layer["w_r"])
    assert B.device_status() == 0


@pytest.mark.parametrize("fp8,values", [(False, False), (True, False), (False, True), (True, True)])
def test_starved_gemm_times_out_and_context_survives(layer, fp8, values):
    L = layer
    if values:
        v, _ = B.quantize_acts_values(L["plan"], L["cb4"], L["x"], fp8=fp8)

        def run(cb_a, cb_w, idx, s, w_idx, w_r):
            return B.qgemm_values(cb_w, v, s, w_idx, w_r, fp8=fp8)
    else:
        run = B.qgemm_fp8 if fp8 else B.qgemm
    ref = run(L["cb4"], L["cb2"], L["idx"], L["s"], L["w_idx"], L["w_r"])
    torch.cuda.synchronize()
    assert B.device_status() == 0
    B.debug_starve(B.OQ_STARVE_GEMM)
    try:
        run(L["cb4"], L["cb2"], L["idx"], L["s"], L["w_idx"], L["w_r"])
        assert B.device_status(clear=True) == 5
    finally:
        _reset_hooks()
    y = run(L["cb4"], L["cb2"], L["idx"], L["s"], L["w_idx"], L["w_r"])
    assert torch.equal(y, ref)
    assert B.device_status() == 0
    # unrelated device work still runs on the context
    a = torch.arange(1000, device=y.device, dtype=torch.float32)
    assert float(a.sum()) == 499500.0


def test_starved_layer_reports_timeout_from_both_kernels(layer):
    L = layer
    B.debug_starve(B.OQ_STARVE_RPBH | B.OQ_STARVE_GEMM)
    try:
        B.qlinear(L["plan"], L["cb4"], L["cb2"], L["x"], L["w_idx"], L["w_r"])
        assert B.device_status(clear=True) == 5
    finally:
        _reset_hooks()
    y = B.qlinear(L["plan"], L["cb4"], L["cb2"], L["x"], L["w_idx"], L["w_r"])
    assert torch.equal(y, L["y"])
    assert B.device_status() == 0


def test_starved_quantizer_releases_the_dependent_gemm(layer):
    """The product launches programmatically after the quantiser and waits
    for it to finish before reading its output.  A quantiser whose waits run
    out still finishes (bounded), so the product's dependency wait ends and
    the layer call returns; the next call is exact again."""
    L = layer
    B.debug_starve(B.OQ_STARVE_RPBH)
    try:
        B.qlinear(L["plan"], L["cb4"], L["cb2"], L["x"], L["w_idx"], L["w_r"])
        assert B.device_status(clear=True) == 5
    finally:
        _reset_hooks()
    y = B.qlinear(L["plan"], L["cb4"], L["cb2"], L["x"], L["w_idx"], L["w_r"])
    assert torch.equal(y, L["y"])
    assert B.device_status() == 0


def test_starved_large_block_quantizer_times_out_and_context_survives(cuda_device):
    """The staged kernel for blocks beyond 128 (Full RHT) bounds its waits too."""
    d = 1024
    plan = B.rotation_plan(d, d, 5, B.OQ_ROT_BLOCK_RHT)
    cb = B.codebook(d, 4)
    x = torch.randn(20, d, device=cuda_device).to(torch.bfloat16)
    ref_idx, ref_s = B.quantize_acts(plan, cb, x)
    torch.cuda.synchronize()
    B.debug_starve(B.OQ_STARVE_RPBH)
    try:
        B.quantize_acts(plan, cb, x)
        assert B.device_status(clear=True) == 5
    finally:
        _reset_hooks()
    idx, s = B.quantize_acts(plan, cb, x)
    assert torch.equal(idx, ref_idx) and torch.equal(s, ref_s)
    assert B.device_status() == 0
