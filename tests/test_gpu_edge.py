"""GPU edge cases of the C ABI: empty and degenerate inputs, non-finite rows,
argument and alignment errors, determinism."""
import numpy as np
import pytest
import torch

import oracle
from rotation_bit_quantization_rpbh_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer(cuda_device):
    d, h = 512, 128
    plan = B.rpbh_plan(d, h, 21)
    return plan, B.codebook(d, 4), B.codebook(d, 2), d


def test_empty_batch_is_a_no_op(layer, cuda_device):
    plan, cb4, cb2, d = layer
    x = torch.zeros((0, d), dtype=torch.bfloat16, device=cuda_device)
    idx, s = B.quantize_acts(plan, cb4, x)
    assert idx.shape == (0, d // 2) and s.shape == (0,)
    W = torch.randn(64, d, device=cuda_device).to(torch.bfloat16)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    y = B.qgemm(cb4, cb2, idx, s, w_idx, w_r)
    assert y.shape == (0, 64)


def test_zero_rows_take_the_middle_cell_and_give_zero_output(layer, cuda_device):
    plan, cb4, cb2, d = layer
    x = torch.randn(40, d, device=cuda_device).to(torch.bfloat16)
    x[[0, 17, 39]] = 0
    idx, s = B.quantize_acts(plan, cb4, x)
    u = B.unpack_indices(idx, d, 4).cpu()
    assert torch.all(u[[0, 17, 39]] == 8)
    assert torch.all(s.cpu()[[0, 17, 39]] == 0)
    W = torch.randn(96, d, device=cuda_device).to(torch.bfloat16)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    y = B.qgemm(cb4, cb2, idx, s, w_idx, w_r).cpu()
    assert torch.all(y[[0, 17, 39]] == 0)
    assert torch.count_nonzero(y[1]) > 0


def test_non_finite_rows_are_quantised_to_the_middle_cell(layer, cuda_device):
    plan, cb4, _, d = layer
    x = torch.randn(8, d, device=cuda_device)
    x[2, 5] = float("inf")
    x[5, 100] = float("nan")
    idx, s = B.quantize_acts(plan, cb4, x)
    u = B.unpack_indices(idx, d, 4).cpu()
    assert torch.all(u[2] == 8) and torch.all(u[5] == 8)
    sc = s.cpu()
    assert not torch.isfinite(sc[2]) and not torch.isfinite(sc[5])
    assert torch.all(torch.isfinite(sc[[0, 1, 3, 4, 6, 7]]))
    assert B.device_status() == 0


def test_misaligned_pointers_are_rejected(layer, cuda_device):
    plan, cb4, _, d = layer
    buf = torch.randn(9 * d + 1, device=cuda_device).to(torch.bfloat16)
    x = buf[1:1 + 8 * d].view(8, d)  # 2-byte offset
    with pytest.raises(B.OQError) as e:
        B.quantize_acts(plan, cb4, x)
    assert e.value.status == 3


def test_mismatched_handles_are_rejected(layer, cuda_device):
    plan, cb4, _, d = layer
    other = B.codebook(256, 4)
    x = torch.randn(4, d, device=cuda_device).to(torch.bfloat16)
    with pytest.raises(B.OQError) as e:
        B.quantize_acts(plan, other, x)
    assert e.value.status == 1
    cb5 = B.codebook(d, 5)  # a codebook width the quantiser does not pack
    with pytest.raises(B.OQError) as e:
        B.quantize_acts(plan, cb5, x)
    assert e.value.status == 2


def test_workspace_too_small_is_reported(layer, cuda_device):
    plan, cb4, cb2, d = layer
    x = torch.randn(16, d, device=cuda_device).to(torch.bfloat16)
    W = torch.randn(32, d, device=cuda_device).to(torch.bfloat16)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    ws = torch.empty(64, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(B.OQError) as e:
        B.qlinear(plan, cb4, cb2, x, w_idx, w_r, workspace=ws)
    assert e.value.status == 6


def test_results_are_deterministic(layer, cuda_device):
    plan, cb4, cb2, d = layer
    x = torch.randn(333, d, device=cuda_device).to(torch.bfloat16)
    W = torch.randn(300, d, device=cuda_device).to(torch.bfloat16)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    y1 = B.qlinear(plan, cb4, cb2, x, w_idx, w_r)
    y2 = B.qlinear(plan, cb4, cb2, x, w_idx, w_r)
    assert torch.equal(y1, y2)


def test_outputs_run_on_a_side_stream(layer, cuda_device):
    plan, cb4, cb2, d = layer
    x = torch.randn(100, d, device=cuda_device).to(torch.bfloat16)
    W = torch.randn(128, d, device=cuda_device).to(torch.bfloat16)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    ref = B.qlinear(plan, cb4, cb2, x, w_idx, w_r)
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        y = B.qlinear(plan, cb4, cb2, x, w_idx, w_r, stream=st)
    torch.cuda.current_stream().wait_stream(st)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)


def test_binding_checks_buffers_before_the_call(layer, cuda_device):
    """Wrong shapes, dtypes, layouts or devices are refused in the binding,
    before the C ABI (which sees only pointers and sizes) could overrun them."""
    plan, cb4, cb2, d = layer
    x = torch.randn(16, d, device=cuda_device).to(torch.bfloat16)
    W = torch.randn(32, d, device=cuda_device).to(torch.bfloat16)
    w_idx, w_r = B.quantize_weights(plan, cb2, W)
    with pytest.raises(ValueError):  # y of the wrong shape
        B.qlinear(plan, cb4, cb2, x, w_idx, w_r, y=torch.empty((16, 31), dtype=torch.bfloat16, device=cuda_device))
    with pytest.raises(ValueError):  # y of the wrong dtype
        B.qlinear_noalloc(plan, cb4, cb2, x, w_idx, w_r, torch.empty((16, 32), dtype=torch.float32,
                                                                   device=cuda_device))
    with pytest.raises(ValueError):  # x not contiguous
        B.quantize_acts(plan, cb4, torch.randn(d, 16, device=cuda_device).to(torch.bfloat16).t())
    with pytest.raises(ValueError):  # x narrower than the plan's d
        B.quantize_acts(plan, cb4, x[:, : d // 2].contiguous())
    with pytest.raises(ValueError):  # packed W rows of another width
        B.qlinear(plan, cb4, cb2, x, w_idx[:, :-1].contiguous(), w_r)
    with pytest.raises(ValueError):  # norms of another dtype
        B.qgemm(cb4, cb2, torch.zeros((16, d // 2), dtype=torch.uint8, device=cuda_device),
                torch.ones(16, dtype=torch.float16, device=cuda_device), w_idx, w_r)
    with pytest.raises(ValueError):  # an output on the host
        B.quantize_acts(plan, cb4, x, s_out=torch.empty(16))


@pytest.mark.parametrize("fp8", [False, True])
def test_layer_replays_in_a_cuda_graph(cuda_device, fp8):
    """The layer call captured in a CUDA graph replays to the same bits as
    the eager call, on new inputs copied into the captured buffer. One eager
    call first uploads the tables and sets the kernels' attributes, which
    capture cannot do. The two launches keep their programmatic dependency
    inside the graph."""
    M, d, N, h = 512, 1536, 768, 128
    plan = B.rpbh_plan(d, h, 5)
    cb_a, cb_w = B.codebook(d, 4), B.codebook(d, 4)
    g = torch.Generator().manual_seed(5)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16).to(cuda_device)
    x1 = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16).to(cuda_device)
    x2 = (torch.randn(M, d, generator=g) * 3.0).to(torch.bfloat16).to(cuda_device)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W)
    need = max(B.qlinear_workspace_values(M, d), B.qlinear_workspace(M, d, 4))
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    xin = x1.clone()
    y = torch.empty((M, N), dtype=torch.bfloat16, device=cuda_device)
    B.qlinear(plan, cb_a, cb_w, xin, w_idx, w_r, y=y, workspace=ws, fp8=fp8)  # eager: uploads, attributes
    torch.cuda.synchronize()
    y1_eager = y.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        B.qlinear(plan, cb_a, cb_w, xin, w_idx, w_r, y=y, workspace=ws, fp8=fp8)
    y.zero_()
    xin.copy_(x2)
    graph.replay()
    torch.cuda.synchronize()
    y2_graph = y.clone()
    xin.copy_(x1)
    graph.replay()
    torch.cuda.synchronize()
    assert B.device_status() == 0
    y2_eager = B.qlinear(plan, cb_a, cb_w, x2, w_idx, w_r, fp8=fp8)
    torch.cuda.synchronize()
    assert torch.equal(y, y1_eager)
    assert torch.equal(y2_graph, y2_eager)
    assert not torch.equal(y2_graph, y1_eager)
    del graph
