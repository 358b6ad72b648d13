"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and its host-side logic (codebook solver, plan generator, argument
checks) agrees with the oracle.  No GPU compute is called here."""
import math
import os
import re

import numpy as np
import pytest

import oracle
from rotation_bit_quantization_rpbh_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "oq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(oq_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = B.lib()
    syms = header_symbols()
    assert len(syms) >= 18
    for s in syms:
        assert hasattr(L, s), s
    assert sorted(B.EXPORTS) == syms


def test_status_strings():
    L = B.lib()
    assert L.oq_status_str(0) == b"OQ_OK"
    assert L.oq_status_str(5) == b"OQ_ERR_TIMEOUT"


@pytest.mark.parametrize("d,bits", [(256, 4), (3072, 4), (12288, 4), (4096, 2), (4096, 4), (1536, 4), (1536, 6),
                                    (64, 2), (64, 4), (64, 6), (512, 2), (8, 2), (3072, 3), (128, 3), (256, 8)])
def test_library_codebook_matches_oracle(d, bits):
    """Two independent solvers (library: Newton on the Lloyd-Max conditions
    with incomplete-beta cell masses; oracle: Lloyd iteration with
    Gauss-Legendre quadrature) land on the same C_d."""
    cb = B.codebook(d, bits)
    c, t = cb.values()
    co, to = oracle.codebook(d, bits)
    assert np.max(np.abs(c - co)) * math.sqrt(d) < 1e-10
    np.testing.assert_array_equal(t.astype(np.float32), to.astype(np.float32))
    assert t[len(t) // 2] == 0.0
    np.testing.assert_array_equal(c, -c[::-1])
    np.testing.assert_array_equal(cb.bf16_bits(), oracle.round_bf16(co)[0])


@pytest.mark.parametrize("d,h,seed", [(256, 64, 0), (3072, 128, 1), (12288, 128, 2), (4096, 128, 3), (1536, 128, 4),
                                      (64, 16, 99)])
def test_library_plan_matches_oracle(d, h, seed):
    p1, s1 = B.rpbh_plan_host(d, h, seed)
    p2, s2 = oracle.plan(d, h, seed)
    np.testing.assert_array_equal(p1, p2)
    np.testing.assert_array_equal(s1, s2)


def test_library_plan_matches_hand_derived_golden():
    """The library's shuffle against the permutation derived by hand from the
    published SplitMix64 outputs (tests/golden), independently of the oracle."""
    import os

    golden = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "fisher_yates_d5_seed1234567.txt")
    with open(golden) as f:
        rows = {ln.split()[0]: ln.split()[1:] for ln in f if ln.strip() and not ln.startswith("#")}
    seed, d = int(rows["seed"][0]), int(rows["d"][0])
    perm, sign = B.rpbh_plan_host(d, d, seed)
    assert perm.tolist() == [int(v) for v in rows["perm"]]
    assert int(sign[0]) == int(rows["sign0"][0])


@pytest.mark.parametrize("d,h,seed", [(256, 64, 0), (4096, 128, 3)])
def test_library_block_rht_plan_matches_oracle(d, h, seed):
    p1, s1 = B.rotation_plan_host(d, h, seed, B.OQ_ROT_BLOCK_RHT)
    p2, s2 = oracle.plan(d, h, seed, variant=oracle.BLOCK_RHT)
    np.testing.assert_array_equal(p1, p2)
    np.testing.assert_array_equal(s1, s2)
    p3, s3 = B.rotation_plan_host(d, h, seed, B.OQ_ROT_RPBH)  # the RPBH variant is oq_rpbh_plan's plan
    p4, s4 = B.rpbh_plan_host(d, h, seed)
    np.testing.assert_array_equal(p3, p4)
    np.testing.assert_array_equal(s3, s4)


@pytest.mark.parametrize("d,bits", [(256, 4), (3072, 4), (4096, 2), (1536, 6), (12288, 4), (3072, 3)])
def test_fp8_centroid_bytes_are_e4m3_of_the_scaled_codebook(d, bits):
    """oq_codebook_fp8: e4m3 (torch's round-to-nearest-even conversion) of
    c_j sqrt(d) for the oracle's fp64 centroids."""
    import math

    import torch

    cb = B.codebook(d, bits)
    c = oracle.codebook(d, bits)[0]
    want = torch.tensor(np.asarray(c) * math.sqrt(d), dtype=torch.float64).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(cb.e4m3_bytes(), want.view(torch.uint8).numpy())


def test_unknown_rotation_variant_is_rejected():
    import ctypes

    L = B.lib()
    perm = np.zeros(256, dtype=np.int32)
    sign = np.zeros(256, dtype=np.int8)
    assert L.oq_rotation_plan_host(256, 64, ctypes.c_uint64(0), 7, perm.ctypes.data_as(ctypes.c_void_p),
                                   sign.ctypes.data_as(ctypes.c_void_p)) == 1


def test_argument_checks_on_host_calls():
    L = B.lib()
    import ctypes

    h = ctypes.c_void_p()
    assert L.oq_codebook(256, 9, ctypes.byref(h)) == 2  # UNSUPPORTED
    assert L.oq_codebook(2, 4, ctypes.byref(h)) == 2
    assert L.oq_codebook(256, 4, None) == 1  # INVALID_ARG
    perm = np.zeros(300, dtype=np.int32)
    sign = np.zeros(300, dtype=np.int8)
    P = perm.ctypes.data_as(ctypes.c_void_p)
    S = sign.ctypes.data_as(ctypes.c_void_p)
    assert L.oq_rpbh_plan_host(300, 128, 0, P, S) == 2  # d % h != 0
    assert L.oq_rpbh_plan_host(256, 96, 0, P, S) == 2  # d % h != 0
    assert L.oq_rpbh_plan_host(256, 256, 0, P, S) == 0  # the host plan's arrays do not depend on h
    assert L.oq_rpbh_plan_host(5, 5, 0, P, S) == 0
    assert L.oq_rpbh_plan_host(40000, 8, 0, P, S) == 2  # beyond the 16-bit gather offsets
    assert L.oq_rpbh_plan_host(0, 64, 0, P, S) == 1
    assert L.oq_rpbh_plan_host(256, 64, 0, P, S) == 0


def test_debug_hooks_leave_host_calls_alone():
    """The failure hooks only touch device allocations and kernel launches:
    host-side plans and codebooks are built while failures are pending."""
    import ctypes

    L = B.lib()
    B.debug_fail_allocations(3)
    B.debug_starve(B.OQ_STARVE_RPBH | B.OQ_STARVE_GEMM)
    try:
        perm = np.zeros(256, dtype=np.int32)
        sign = np.zeros(256, dtype=np.int8)
        assert L.oq_rpbh_plan_host(256, 64, 3, perm.ctypes.data_as(ctypes.c_void_p),
                                   sign.ctypes.data_as(ctypes.c_void_p)) == 0
        assert sorted(perm.tolist()) == list(range(256))
        cb = B.codebook(256, 4)
        assert cb.bits == 4
    finally:
        B.debug_fail_allocations(0)
        B.debug_starve(0)


def test_workspace_size():
    ws = B.qlinear_workspace(4096, 3072, 4)
    assert ws >= 4096 * 1536 + 4096 * 4 and ws % 256 == 0
    assert B.qlinear_workspace(32760, 1536, 6) >= 32760 * 1536 + 32760 * 4
    assert B.qlinear_workspace(0, 1536, 4) == 0
    ws3 = B.qlinear_workspace(10, 1536, 3)  # 3-bit: 8 codes per 3 bytes
    assert ws3 >= 10 * 1536 * 3 // 8 + 10 * 4 and ws3 % 256 == 0
    assert B.qlinear_workspace(10, 1536, 5) == 0
    assert B.qlinear_workspace(10, 1536, 8) >= 10 * 1536 + 10 * 4  # 8-bit: one byte per code
    wv = B.qlinear_workspace_values(4096, 3072)
    assert wv >= 4096 * 3072 * 2 + 4096 * 4 and wv % 256 == 0


def test_unpack_layout():
    import torch

    # two 4-bit codes per byte, LSB first; four 2-bit codes per byte
    p4 = torch.tensor([[0x21, 0x43]], dtype=torch.uint8)
    assert B.unpack_indices(p4, 4, 4).tolist() == [[1, 2, 3, 4]]
    p2 = torch.tensor([[0b11100100]], dtype=torch.uint8)
    assert B.unpack_indices(p2, 4, 2).tolist() == [[0, 1, 2, 3]]
    p6 = torch.tensor([[63, 5]], dtype=torch.uint8)
    assert B.unpack_indices(p6, 2, 6).tolist() == [[63, 5]]
    p8 = torch.tensor([[255, 0, 128]], dtype=torch.uint8)
    assert B.unpack_indices(p8, 3, 8).tolist() == [[255, 0, 128]]
    # 3-bit: a bit stream, code k in bits 3k..3k+2 of the row (LSB first):
    # codes 0..7 = 0,1,...,7 -> bits 000 001 010 011 100 101 110 111 from bit 0
    stream = sum(k << (3 * k) for k in range(8))  # 24 bits
    p3 = torch.tensor([[stream & 0xFF, (stream >> 8) & 0xFF, stream >> 16]], dtype=torch.uint8)
    assert B.unpack_indices(p3, 8, 3).tolist() == [list(range(8))]
    assert B.packed_row_bytes(1536, 8) == 1536 and B.packed_row_bytes(1536, 6) == 1536


def test_binding_rejects_buffers_the_kernels_would_overrun():
    """The C ABI sees only pointers and sizes, so the binding checks shapes,
    dtypes, layout and device before any call (ValueError, no library call)."""
    import torch

    class FakePlan:  # only the dimension is read before the checks fail
        d = 256
        handle = None

    class FakeCb:
        d, bits = 256, 4
        handle = None

    x_cpu = torch.zeros((8, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.quantize_acts(FakePlan(), FakeCb(), x_cpu)  # not on a CUDA device
    with pytest.raises(ValueError):
        B.quantize_weights(FakePlan(), FakeCb(), torch.zeros((8, 256)))
    with pytest.raises(ValueError):
        B.rpbh_apply(FakePlan(), torch.zeros(256))  # not 2-D
    with pytest.raises(ValueError):
        B.qlinear(FakePlan(), FakeCb(), FakeCb(), x_cpu, torch.zeros((4, 128), dtype=torch.uint8),
                  torch.zeros(4, dtype=torch.bfloat16))
    assert B.packed_row_bytes(256, 3) == 96 and B.packed_row_bytes(256, 6) == 256
    assert B.packed_row_bytes(256, 8) == 256 and B.packed_row_bytes(256, 2) == 64
