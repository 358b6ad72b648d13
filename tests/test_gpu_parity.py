"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs -- multi-tile ragged cases checked in full; at the
five workload shapes at full size, the codes and norms of every activation
and weight row, the rotation on 512 rows, and the product on 512 rows x all
N plus all M x 256 columns.

Tolerances are stated in tests/parity.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from rotation_bit_quantization_rpbh_b200 import binding as B
from rotation_bit_quantization_rpbh_b200 import inputs as I

from parity import (GEMM_TOL, check_product, check_quantized_rows, check_rotation, gemm_reference, rel_frob,
                    stored_oracle_codebook, to_f64)

pytestmark = pytest.mark.gpu


def _run_layer(dev, M, d, N, h, bw, ba, x_cpu, W_cpu, seed, full_check, n_rot=512, n_rows_gemm=512, n_cols_gemm=256,
               bias=False):
    rng = np.random.default_rng(seed + 7)
    plan = B.rpbh_plan(d, h, seed)
    perm, sign = oracle.plan(d, h, seed)
    pe, se = plan.export()
    np.testing.assert_array_equal(pe, perm)
    np.testing.assert_array_equal(se, sign)
    cb_a, cb_w = B.codebook(d, ba), B.codebook(d, bw)
    ocb_a, ocb_w = oracle.codebook(d, ba), oracle.codebook(d, bw)

    xg, Wg = x_cpu.to(dev), W_cpu.to(dev)
    w_idx, w_r = B.quantize_weights(plan, cb_w, Wg)
    a_idx, s = B.quantize_acts(plan, cb_a, xg)
    bias_t = None
    if bias:
        bias_t = (torch.randn(N, generator=torch.Generator().manual_seed(seed)) * 0.1).to(torch.bfloat16).to(dev)
    y = B.qgemm(cb_a, cb_w, a_idx, s, w_idx, w_r, bias=bias_t)
    y2 = B.qlinear(plan, cb_a, cb_w, xg, w_idx, w_r, bias=bias_t)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    # the one-call layer is the two calls it is made of
    assert torch.equal(y, y2)
    _check_values_schedule(dev, plan, cb_a, cb_w, xg, a_idx, s, w_idx, w_r, bias_t, y, ba, bw, fp8=False)

    # codes and norms of every row of x and of W
    rot_rows = np.arange(M) if full_check else np.sort(rng.choice(M, min(M, n_rot), replace=False))
    check_rotation(plan, x_cpu, rot_rows, h, perm, sign, dev)
    nb_a, _ = check_quantized_rows(a_idx, s, x_cpu, np.arange(M), h, perm, sign, cb_a, ocb_a, "acts")
    nb_w, n_ulp = check_quantized_rows(w_idx, w_r, W_cpu, np.arange(N), h, perm, sign, cb_w, ocb_w, "weights")

    # product: oracle fp64 on the GPU's indices, norms and the bf16 centroid values
    ia = B.unpack_indices(a_idx, d, ba).cpu().numpy()
    iw = B.unpack_indices(w_idx, d, bw).cpu().numpy()
    s64 = s.cpu().numpy().astype(np.float64)
    r64 = w_r.cpu().to(torch.float32).numpy().astype(np.float64)
    ca = oracle.round_bf16(ocb_a[0])[1]
    cw = oracle.round_bf16(ocb_w[0])[1]
    np.testing.assert_array_equal(oracle.round_bf16(ocb_a[0])[0], cb_a.bf16_bits())
    yg = y.cpu().to(torch.float32).numpy().astype(np.float64)
    b64 = None if bias_t is None else bias_t.cpu().to(torch.float32).numpy().astype(np.float64)
    if full_check:
        ref = gemm_reference(ia, s64, iw, r64, ca, cw)
        if b64 is not None:
            ref = ref + b64[None, :]
        err, _, worst = check_product(yg, ref)
    else:
        rr = np.sort(rng.choice(M, min(M, n_rows_gemm), replace=False))
        cc = np.sort(rng.choice(N, min(N, n_cols_gemm), replace=False))
        ref_r = gemm_reference(ia, s64, iw, r64, ca, cw, rows=rr)
        ref_c = gemm_reference(ia, s64, iw, r64, ca, cw, cols=cc)
        if b64 is not None:
            ref_r = ref_r + b64[None, :]
            ref_c = ref_c + b64[None, cc]
        e1, _, w1 = check_product(yg[rr], ref_r)
        e2, _, w2 = check_product(yg[:, cc], ref_c)
        err, worst = max(e1, e2), max(w1, w2)
    return {"band_a": nb_a, "band_w": nb_w, "coords_a": M * d, "coords_w": N * d, "r_ulp": n_ulp, "gemm_rel": err,
            "worst_elem_over_bound": worst}


def _check_values_schedule(dev, plan, cb_a, cb_w, xg, a_idx, s, w_idx, w_r, bias_t, y, ba, bw, fp8):
    """The values schedule against the codes one: the quantiser's values are
    the codebook's values at the codes' indices (same norms), and the product
    from those values equals the product from the codes bit for bit."""
    d = xg.shape[1]
    val, s_v = B.quantize_acts_values(plan, cb_a, xg, fp8=fp8)
    u = B.unpack_indices(a_idx, d, ba).long()
    if fp8:
        tab = torch.from_numpy(cb_a.e4m3_bytes()).to(dev)
        assert torch.equal(val, tab[u])
    else:
        tab = torch.from_numpy(cb_a.bf16_bits().view(np.int16)).to(dev)
        assert torch.equal(val.view(torch.int16), tab[u])
    assert torch.equal(s_v, s)
    if bw == 3 and not fp8:
        return
    y3 = B.qgemm_values(cb_w, val, s_v, w_idx, w_r, bias=bias_t, fp8=fp8)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.equal(y3, y)


# multi-tile cases with ragged edges, checked in full
SMALL = [
    # M,   d,   N,  h, bw, ba, dtype, seed, bias
    (300, 512, 520, 128, 4, 4, "bf16", 11, False),   # 3 M tiles (ragged), 3 N tiles (ragged), 8 K steps
    (129, 256, 200, 64, 2, 4, "f32", 12, True),     # ragged M by one row, N below one tile
    (77, 384, 264, 128, 4, 6, "bf16", 13, False),   # 6-bit activations, 1 byte per code
    (1, 64, 8, 16, 2, 2, "bf16", 14, False),        # a single row, one K step, tiny N
    (260, 1024, 256, 32, 6, 2, "f32", 15, True),    # 6-bit weights, 2-bit activations, h = 32
    (513, 768, 272, 128, 2, 6, "bf16", 16, False),
    (70, 256, 131, 64, 4, 4, "bf16", 17, True),     # N not a multiple of 8: unaligned output rows
]


@pytest.mark.parametrize("case", SMALL, ids=[f"M{c[0]}_d{c[1]}_N{c[2]}_h{c[3]}_W{c[4]}A{c[5]}_{c[6]}" for c in SMALL])
def test_small_layers_match_oracle_in_full(cuda_device, case):
    M, d, N, h, bw, ba, dt, seed, bias = case
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))
    x[:, torch.randint(0, d, (3,), generator=g)] *= 30.0
    W = torch.randn(N, d, generator=g) * 0.02
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    _run_layer(cuda_device, M, d, N, h, bw, ba, x.to(dtype), W.to(dtype), seed, full_check=True, bias=bias)


@pytest.mark.parametrize("name", I.ORDER)
def test_workload_at_full_size(cuda_device, name):
    w = I.WORKLOADS[name]
    x = I.make_x(w)
    W = I.make_w(w)
    full = name == "tiny_w4a4"
    stats = _run_layer(cuda_device, w.M, w.d, w.N, w.h, w.bits_w, w.bits_a, x, W, w.plan_seed, full_check=full)
    print(name, stats)


@pytest.mark.parametrize("M,d,h,ba,dt", [(300, 512, 128, 4, "bf16"), (96, 1536, 128, 6, "bf16"),
                                         (130, 256, 64, 2, "f32"), (77, 3072, 128, 4, "bf16")])
def test_block_rht_variant_matches_oracle(cuda_device, M, d, h, ba, dt):
    """The rotation ablation's Block-RHT plan (no permutation; each block is
    read contiguously): rotation, norms and codes against the oracle's
    variant, and the value outputs equal to the codebook at the codes."""
    plan = B.rotation_plan(d, h, 21, B.OQ_ROT_BLOCK_RHT)
    perm, sign = oracle.plan(d, h, 21, variant=oracle.BLOCK_RHT)
    pe, se = plan.export()
    np.testing.assert_array_equal(pe, perm)
    np.testing.assert_array_equal(se, sign)
    g = torch.Generator().manual_seed(21)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g)))
    x = x.to(torch.bfloat16 if dt == "bf16" else torch.float32)
    cb_a, ocb_a = B.codebook(d, ba), oracle.codebook(d, ba)
    a_idx, s = B.quantize_acts(plan, cb_a, x.to(cuda_device))
    val, s_v = B.quantize_acts_values(plan, cb_a, x.to(cuda_device))
    torch.cuda.synchronize()
    assert B.device_status() == 0
    rows = np.arange(M)
    check_rotation(plan, x, rows, h, perm, sign, cuda_device)
    check_quantized_rows(a_idx, s, x, rows, h, perm, sign, cb_a, ocb_a, "acts")
    u = B.unpack_indices(a_idx, d, ba).long()
    tab = torch.from_numpy(cb_a.bf16_bits().view(np.int16)).to(cuda_device)
    assert torch.equal(val.view(torch.int16), tab[u]) and torch.equal(s_v, s)


@pytest.mark.parametrize("M,d,h,variant,ba,dt", [
    (70, 4096, 4096, "block_rht", 4, "bf16"),   # Full RHT: one Walsh-Hadamard block over d
    (33, 1024, 1024, "block_rht", 2, "f32"),
    (50, 3072, 1024, "block_rht", 6, "bf16"),   # the largest power-of-two block of d = 3 * 1024
    (41, 2048, 512, "rpbh", 4, "bf16"),        # RPBH with blocks larger than the in-register kernel
    (9, 16384, 16384, "block_rht", 4, "bf16"),
])
def test_large_block_rotation_matches_oracle(cuda_device, M, d, h, variant, ba, dt):
    """Blocks of h > 128 (the rotation ablation's Full RHT, h = d) run in the
    staged kernel: rotation, norms and codes against the oracle's direct
    O(h) sums, and the value outputs equal to the codebook at the codes."""
    seed = 70 + M
    v = B.OQ_ROT_BLOCK_RHT if variant == "block_rht" else B.OQ_ROT_RPBH
    plan = B.rotation_plan(d, h, seed, v)
    perm, sign = oracle.plan(d, h, seed, variant=oracle.BLOCK_RHT if variant == "block_rht" else 0)
    pe, se = plan.export()
    np.testing.assert_array_equal(pe, perm)
    np.testing.assert_array_equal(se, sign)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))
    x[:, torch.randint(0, d, (4,), generator=g)] *= 25.0
    x = x.to(torch.bfloat16 if dt == "bf16" else torch.float32)
    cb_a, ocb_a = B.codebook(d, ba), oracle.codebook(d, ba)
    xg = x.to(cuda_device)
    a_idx, s = B.quantize_acts(plan, cb_a, xg)
    val, s_v = B.quantize_acts_values(plan, cb_a, xg)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    rows = np.arange(M)
    check_rotation(plan, x, rows, h, perm, sign, cuda_device)
    check_quantized_rows(a_idx, s, x, rows, h, perm, sign, cb_a, ocb_a, "acts")
    u = B.unpack_indices(a_idx, d, ba).long()
    tab = torch.from_numpy(cb_a.bf16_bits().view(np.int16)).to(cuda_device)
    assert torch.equal(val.view(torch.int16), tab[u])
    assert torch.equal(s_v, s)


def _e4m3_values(c, d):
    """e4m3 centroid values of the fp8 variant, from the oracle's fp64 codebook:
    c_j sqrt(d) rounded once to e4m3 (torch's conversion), scaled back."""
    q = torch.tensor(np.asarray(c) * math.sqrt(d), dtype=torch.float64).to(torch.float8_e4m3fn)
    return q.to(torch.float64).numpy() / math.sqrt(d)


FP8_CASES = [
    # M,   d,   N,  h, bw, ba, seed, bias
    (300, 512, 520, 128, 4, 4, 41, False),
    (129, 256, 200, 64, 2, 4, 42, True),
    (77, 384, 264, 128, 4, 6, 43, False),
    (260, 1024, 256, 32, 6, 2, 44, True),
    (70, 256, 131, 64, 4, 4, 45, True),
]


@pytest.mark.parametrize("case", FP8_CASES, ids=[f"M{c[0]}_d{c[1]}_N{c[2]}_W{c[4]}A{c[5]}" for c in FP8_CASES])
def test_fp8_variant_matches_oracle_on_e4m3_centroids(cuda_device, case):
    """The fp8 GEMM variant against the oracle's fp64 product on the same
    indices and norms and the e4m3 centroid values, checked in full."""
    M, d, N, h, bw, ba, seed, bias = case
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16)
    plan = B.rpbh_plan(d, h, seed)
    cb_a, cb_w = B.codebook(d, ba), B.codebook(d, bw)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W.to(cuda_device))
    a_idx, s = B.quantize_acts(plan, cb_a, x.to(cuda_device))
    bias_t = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16).to(cuda_device) if bias else None
    y = B.qgemm_fp8(cb_a, cb_w, a_idx, s, w_idx, w_r, bias=bias_t)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    _check_values_schedule(cuda_device, plan, cb_a, cb_w, x.to(cuda_device), a_idx, s, w_idx, w_r, bias_t, y, ba, bw,
                           fp8=True)
    ca = _e4m3_values(oracle.codebook(d, ba)[0], d)
    cw = _e4m3_values(oracle.codebook(d, bw)[0], d)
    ia = B.unpack_indices(a_idx, d, ba).cpu().numpy()
    iw = B.unpack_indices(w_idx, d, bw).cpu().numpy()
    ref = gemm_reference(ia, s.cpu().numpy().astype(np.float64), iw,
                         w_r.cpu().to(torch.float32).numpy().astype(np.float64), ca, cw)
    if bias:
        ref = ref + bias_t.cpu().to(torch.float32).numpy().astype(np.float64)[None, :]
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    check_product(got, ref)


def test_fp8_variant_needs_d_multiple_of_128(cuda_device):
    d = 64
    cb = B.codebook(d, 4)
    a_idx = torch.zeros((8, d // 2), dtype=torch.uint8, device=cuda_device)
    s = torch.ones(8, device=cuda_device)
    w_idx = torch.zeros((16, d // 2), dtype=torch.uint8, device=cuda_device)
    w_r = torch.ones(16, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(B.OQError) as e:
        B.qgemm_fp8(cb, cb, a_idx, s, w_idx, w_r)
    assert e.value.status == 2  # OQ_ERR_UNSUPPORTED


def test_fp8_variant_full_size_flux_qkv_sample(cuda_device):
    """FLUX-QKV shape in the launch configuration the bench times, checked on
    sampled rows and columns."""
    w = I.WORKLOADS["flux_qkv_w4a4"]
    x = I.make_x(w)
    W = I.make_w(w)
    plan = B.rpbh_plan(w.d, w.h, w.plan_seed)
    cb_a, cb_w = B.codebook(w.d, w.bits_a), B.codebook(w.d, w.bits_w)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W.to(cuda_device))
    a_idx, s = B.quantize_acts(plan, cb_a, x.to(cuda_device))
    y = B.qgemm_fp8(cb_a, cb_w, a_idx, s, w_idx, w_r)
    torch.cuda.synchronize()
    _check_values_schedule(cuda_device, plan, cb_a, cb_w, x.to(cuda_device), a_idx, s, w_idx, w_r, None, y,
                           w.bits_a, w.bits_w, fp8=True)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(w.M, 128, replace=False))
    cols = np.sort(rng.choice(w.N, 256, replace=False))
    ca = _e4m3_values(oracle.codebook(w.d, w.bits_a)[0], w.d)
    cw = _e4m3_values(oracle.codebook(w.d, w.bits_w)[0], w.d)
    ia = B.unpack_indices(a_idx, w.d, w.bits_a).cpu().numpy()
    iw = B.unpack_indices(w_idx, w.d, w.bits_w).cpu().numpy()
    ref = gemm_reference(ia, s.cpu().numpy().astype(np.float64), iw,
                         w_r.cpu().to(torch.float32).numpy().astype(np.float64), ca, cw, rows, cols)
    got = y.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)]
    check_product(got, ref)


@pytest.mark.parametrize("M,d,h,seed", [(300, 512, 128, 51), (97, 384, 64, 52), (64, 256, 32, 53)])
def test_three_bit_codes_match_oracle(cuda_device, M, d, h, seed):
    """3-bit codes (8 per 3 bytes, LSB first) for activations and weights."""
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    plan = B.rpbh_plan(d, h, seed)
    perm, sign = oracle.plan(d, h, seed)
    cb, ocb = B.codebook(d, 3), oracle.codebook(d, 3)
    a_idx, s = B.quantize_acts(plan, cb, x.to(cuda_device))
    w_idx, r = B.quantize_weights(plan, cb, x.to(cuda_device))
    torch.cuda.synchronize()
    assert a_idx.shape == (M, d * 3 // 8)
    rows = np.arange(M)
    check_quantized_rows(a_idx, s, x, rows, h, perm, sign, cb, ocb, "acts")
    check_quantized_rows(w_idx, r, x, rows, h, perm, sign, cb, ocb, "weights")


@pytest.mark.parametrize("bw,ba", [(3, 3), (4, 3), (3, 4)])
def test_three_bit_fp8_product_matches_oracle(cuda_device, bw, ba):
    """W3A3 (the pages' ablation setting) and the mixed 3/4-bit pairs through
    the fp8 variant, against the oracle on the e4m3 centroid values."""
    M, d, N, h, seed = 260, 768, 264, 128, 54 + bw + ba
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16)
    plan = B.rpbh_plan(d, h, seed)
    cb_a, cb_w = B.codebook(d, ba), B.codebook(d, bw)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W.to(cuda_device))
    xg = x.to(cuda_device)
    a_idx, s = B.quantize_acts(plan, cb_a, xg)
    y = B.qgemm_fp8(cb_a, cb_w, a_idx, s, w_idx, w_r)
    y2 = B.qlinear(plan, cb_a, cb_w, xg, w_idx, w_r, fp8=True)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.equal(y, y2)
    ca = _e4m3_values(oracle.codebook(d, ba)[0], d)
    cw = _e4m3_values(oracle.codebook(d, bw)[0], d)
    ia = B.unpack_indices(a_idx, d, ba).cpu().numpy()
    iw = B.unpack_indices(w_idx, d, bw).cpu().numpy()
    ref = gemm_reference(ia, s.cpu().numpy().astype(np.float64), iw,
                         w_r.cpu().to(torch.float32).numpy().astype(np.float64), ca, cw)
    check_product(y.float().cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("bw,ba", [(3, 3), (3, 4), (4, 3)])
def test_three_bit_bf16_product_matches_oracle(cuda_device, bw, ba):
    """W3A3 (a setting of the page's ablation) and the mixed 3/4-bit pairs at
    the bf16 centroid precision the rest of the layer uses: the codes product,
    the values product and the one-call layer against the oracle's fp64
    product on the same indices, norms and bf16 centroids."""
    M, d, N, h, seed = 300, 768, 520, 128, 64 + bw + ba
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16)
    plan = B.rpbh_plan(d, h, seed)
    cb_a, cb_w = B.codebook(d, ba), B.codebook(d, bw)
    ocb_a, ocb_w = oracle.codebook(d, ba), oracle.codebook(d, bw)
    xg = x.to(cuda_device)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W.to(cuda_device))
    a_idx, s = B.quantize_acts(plan, cb_a, xg)
    bias_t = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16).to(cuda_device)
    y = B.qgemm(cb_a, cb_w, a_idx, s, w_idx, w_r, bias=bias_t)
    y2 = B.qlinear(plan, cb_a, cb_w, xg, w_idx, w_r, bias=bias_t)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.equal(y, y2)
    _check_values_schedule(cuda_device, plan, cb_a, cb_w, xg, a_idx, s, w_idx, w_r, bias_t, y, ba, bw, fp8=False)
    ia = B.unpack_indices(a_idx, d, ba).cpu().numpy()
    iw = B.unpack_indices(w_idx, d, bw).cpu().numpy()
    ca, cw = oracle.round_bf16(ocb_a[0])[1], oracle.round_bf16(ocb_w[0])[1]
    ref = gemm_reference(ia, s.cpu().numpy().astype(np.float64), iw,
                         w_r.cpu().to(torch.float32).numpy().astype(np.float64), ca, cw)
    ref = ref + bias_t.cpu().to(torch.float32).numpy().astype(np.float64)[None, :]
    check_product(y.float().cpu().numpy().astype(np.float64), ref)


def test_values_schedule_limits_are_reported(cuda_device):
    cb3 = B.codebook(192, 3)  # 3-bit rows need d % 128 == 0
    val = torch.zeros((8, 192), dtype=torch.bfloat16, device=cuda_device)
    s = torch.ones(8, device=cuda_device)
    w_idx = torch.zeros((16, 72), dtype=torch.uint8, device=cuda_device)
    w_r = torch.ones(16, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(B.OQError) as e:
        B.qgemm_values(cb3, val, s, w_idx, w_r)
    assert e.value.status == 2
    plan = B.rpbh_plan(192, 64, 3)
    with pytest.raises(B.OQError) as e:  # e4m3 values need d % 128 == 0
        B.quantize_acts_values(plan, B.codebook(192, 4), torch.zeros((4, 192), device=cuda_device), fp8=True)
    assert e.value.status == 2
    bad = torch.zeros(8 * 256 + 8, dtype=torch.bfloat16, device=cuda_device)[1:1 + 8 * 256].view(8, 256)
    w4 = torch.zeros((16, 128), dtype=torch.uint8, device=cuda_device)
    s8 = torch.ones(8, device=cuda_device)
    with pytest.raises(B.OQError) as e:  # values not 16-byte aligned
        B.qgemm_values(B.codebook(256, 4), bad, s8, w4, w_r)
    assert e.value.status == 3


def test_three_bit_limits_are_reported(cuda_device):
    d = 256
    cb = B.codebook(d, 3)
    x = torch.randn(8, d, device=cuda_device).to(torch.bfloat16)
    with pytest.raises(B.OQError) as e:  # h = 16 would give 6-byte blocks
        B.quantize_acts(B.rpbh_plan(d, 16, 1), cb, x)
    assert e.value.status == 2
    a_idx, s = B.quantize_acts(B.rpbh_plan(d, 64, 1), cb, x)
    cb2 = B.codebook(d, 2)
    w_idx = torch.zeros((16, d // 4), dtype=torch.uint8, device=cuda_device)
    w_r = torch.ones(16, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(B.OQError) as e:  # 3-bit codes pair with 3- or 4-bit codes only
        B.qgemm(cb, cb2, a_idx, s, w_idx, w_r)
    assert e.value.status == 2


def test_eight_bit_activations_match_oracle(cuda_device):
    """8-bit activation codes (one byte each) against the oracle, then the W4A8
    layer, which runs in the values schedule (the codes product has no 8-bit
    decoder), against the oracle's product on the same indices: bf16 and fp8."""
    M, d, N, h, seed = 300, 256, 264, 64, 61
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16)
    plan = B.rpbh_plan(d, h, seed)
    perm, sign = oracle.plan(d, h, seed)
    cb_a, cb_w = B.codebook(d, 8), B.codebook(d, 4)
    ocb_a, ocb_w = oracle.codebook(d, 8), oracle.codebook(d, 4)
    xg = x.to(cuda_device)
    a_idx, s = B.quantize_acts(plan, cb_a, xg)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W.to(cuda_device))
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert a_idx.shape == (M, d)
    check_quantized_rows(a_idx, s, x, np.arange(M), h, perm, sign, cb_a, ocb_a, "acts")
    with pytest.raises(B.OQError) as e:
        B.qgemm(cb_a, cb_w, a_idx, s, w_idx, w_r)
    assert e.value.status == 2  # no in-kernel 8-bit decoder
    with pytest.raises(B.OQError) as e:  # a codes-sized workspace leaves only the codes schedule
        B.qlinear(plan, cb_a, cb_w, xg, w_idx, w_r, schedule="codes")
    assert e.value.status == 2

    ia = B.unpack_indices(a_idx, d, 8).cpu().numpy()
    iw = B.unpack_indices(w_idx, d, 4).cpu().numpy()
    s64 = s.cpu().numpy().astype(np.float64)
    r64 = w_r.cpu().to(torch.float32).numpy().astype(np.float64)
    for fp8 in (False, True):
        y = B.qlinear(plan, cb_a, cb_w, xg, w_idx, w_r, fp8=fp8)
        torch.cuda.synchronize()
        assert B.device_status() == 0
        _check_values_schedule(cuda_device, plan, cb_a, cb_w, xg, a_idx, s, w_idx, w_r, None, y, 8, 4, fp8=fp8)
        if fp8:
            ca, cw = _e4m3_values(ocb_a[0], d), _e4m3_values(ocb_w[0], d)
        else:
            ca, cw = oracle.round_bf16(ocb_a[0])[1], oracle.round_bf16(ocb_w[0])[1]
        ref = gemm_reference(ia, s64, iw, r64, ca, cw)
        check_product(y.float().cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("M,d,N,bw,fp8", [(300, 512, 520, 4, False), (700, 256, 264, 2, False),
                                          (513, 384, 200, 6, False), (257, 512, 136, 4, True),
                                          (1100, 768, 512, 3, False)])
def test_tall_tiles_give_the_same_product(cuda_device, M, d, N, bw, fp8):
    """The A-values product in 512-row tiles (two A boxes per decoded W
    stage, both accumulators) against 256-row tiles: the same MMAs in the
    same order per output element, so the same bits; ragged M and N."""
    g = torch.Generator().manual_seed(M + N)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16)
    plan = B.rpbh_plan(d, 128, 7)
    cb_a, cb_w = B.codebook(d, 4), B.codebook(d, bw)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W.to(cuda_device))
    val, s = B.quantize_acts_values(plan, cb_a, x.to(cuda_device), fp8=fp8)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16).to(cuda_device)
    try:
        B.debug_qgemm_tile_rows(256)
        y1 = B.qgemm_values(cb_w, val, s, w_idx, w_r, bias=bias, fp8=fp8)
        B.debug_qgemm_tile_rows(512)
        y2 = B.qgemm_values(cb_w, val, s, w_idx, w_r, bias=bias, fp8=fp8)
    finally:
        B.debug_qgemm_tile_rows(0)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.equal(y1, y2)


def _offset16(t):
    """An empty tensor shaped and typed like t whose data starts 16 bytes past
    a 32-byte boundary (the rows' pitch keeps every row so)."""
    nbytes = t.numel() * t.element_size()
    raw = torch.empty(nbytes + 64, dtype=torch.uint8, device=t.device)
    off = (-raw.data_ptr()) % 32 + 16
    out = raw[off:off + nbytes].view(t.dtype).view(t.shape)
    assert out.data_ptr() % 32 == 16
    return out


# (kernel family, team layout (rows per warp, slots, lanes per block) or None)
_FAMILIES = [(B.RPBH_KERNEL_GROUPS, None), (B.RPBH_KERNEL_TEAMS, None), (B.RPBH_KERNEL_TEAMS, (1, 1, 1)),
             (B.RPBH_KERNEL_TEAMS, (8, 2, 1)), (B.RPBH_KERNEL_TEAMS, (4, 2, 2))]


@pytest.mark.parametrize("family,layout", _FAMILIES)
@pytest.mark.parametrize("M,d,h,ba,dt", [(301, 1536, 128, 4, "bf16"), (130, 256, 64, 2, "f32"),
                                         (77, 3072, 128, 3, "bf16"), (45, 640, 32, 6, "bf16")])
def test_kernel_families_match_oracle(cuda_device, family, layout, M, d, h, ba, dt):
    """Both rotate-and-quantise kernel families (warp groups; teams under
    several forced work layouts) against the oracle on the same ragged
    inputs: rotation and norms, codes for activations and weights, and the
    value outputs equal to the codebook at the codes."""
    g = torch.Generator().manual_seed(d + M)
    x = torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))
    x = x.to(torch.bfloat16 if dt == "bf16" else torch.float32)
    plan = B.rpbh_plan(d, h, 33)
    perm, sign = oracle.plan(d, h, 33)
    cb, ocb = B.codebook(d, ba), oracle.codebook(d, ba)
    xg = x.to(cuda_device)
    try:
        B.debug_rpbh_kernel(family)
        if layout:
            B.debug_rpbh_layout(*layout)
        a_idx, s = B.quantize_acts(plan, cb, xg)
        w_idx, r = B.quantize_weights(plan, cb, xg)
        # the same outputs into buffers 16 but not 32 bytes aligned (16-byte stores)
        a_idx16 = _offset16(a_idx)
        B.quantize_acts(plan, cb, xg, a_idx16)
        val = None
        if ba != 3:
            val, s_v = B.quantize_acts_values(plan, cb, xg)
            val16 = _offset16(val)
            B.quantize_acts_values(plan, cb, xg, val16)
        rows = np.arange(M)
        check_rotation(plan, x, rows, h, perm, sign, cuda_device)
        torch.cuda.synchronize()
    finally:
        B.debug_rpbh_kernel(0)
        B.debug_rpbh_layout(0, 0, 0)
    assert B.device_status() == 0
    assert torch.equal(a_idx16, a_idx)
    if val is not None:
        assert torch.equal(val16, val)
    check_quantized_rows(a_idx, s, x, rows, h, perm, sign, cb, ocb, "acts")
    check_quantized_rows(w_idx, r, x, rows, h, perm, sign, cb, ocb, "weights")
    if val is not None:
        u = B.unpack_indices(a_idx, d, ba).long()
        tab = torch.from_numpy(cb.bf16_bits().view(np.int16)).to(cuda_device)
        assert torch.equal(val.view(torch.int16), tab[u]) and torch.equal(s_v, s)


@pytest.mark.parametrize("M,d,h,variant", [(64, 3072, 128, "rpbh"),        # warp-group kernel
                                           (40, 12288, 128, "rpbh"),       # team kernel, 112 KB table
                                           (48, 1536, 128, "block_rht"),   # team kernel, contiguous reads
                                           (12, 4096, 4096, "block_rht")])  # staged kernel (Full RHT)
def test_eight_bit_codes_in_every_kernel_family(cuda_device, M, d, h, variant):
    """8-bit codes (256 levels: the widest table, which grows with sqrt(d))
    through each kernel family at sizes where the table is large, against
    the oracle; the value outputs equal the codebook at the codes."""
    seed = 90 + M
    v = B.OQ_ROT_BLOCK_RHT if variant == "block_rht" else B.OQ_ROT_RPBH
    plan = B.rotation_plan(d, h, seed, v)
    perm, sign = oracle.plan(d, h, seed, variant=oracle.BLOCK_RHT if variant == "block_rht" else 0)
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16)
    cb, ocb = B.codebook(d, 8), stored_oracle_codebook(d, 8)
    xg = x.to(cuda_device)
    a_idx, s = B.quantize_acts(plan, cb, xg)
    w_idx, r = B.quantize_weights(plan, cb, xg)
    val, s_v = B.quantize_acts_values(plan, cb, xg)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert a_idx.shape == (M, d)
    rows = np.arange(M)
    check_quantized_rows(a_idx, s, x, rows, h, perm, sign, cb, ocb, "acts")
    check_quantized_rows(w_idx, r, x, rows, h, perm, sign, cb, ocb, "weights")
    tab = torch.from_numpy(cb.bf16_bits().view(np.int16)).to(cuda_device)
    assert torch.equal(val.view(torch.int16), tab[a_idx.long()]) and torch.equal(s_v, s)


@pytest.mark.parametrize("fp8", [False, True])
def test_product_gives_the_same_bits_for_every_output_alignment(cuda_device, fp8):
    """The product's epilogue writes 32-byte sectors when y's base and row
    pitch are 32-byte aligned, 16-byte stores otherwise: the same bits."""
    M, d, N, h = 300, 512, 768, 128
    plan = B.rpbh_plan(d, h, 17)
    cb_a, cb_w = B.codebook(d, 4), B.codebook(d, 4)
    g = torch.Generator().manual_seed(17)
    x = (torch.randn(M, d, generator=g) * torch.exp(torch.randn(d, generator=g))).to(torch.bfloat16).to(cuda_device)
    W = (torch.randn(N, d, generator=g) * 0.02).to(torch.bfloat16).to(cuda_device)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W)
    val, s = B.quantize_acts_values(plan, cb_a, x, fp8=fp8)
    y = B.qgemm_values(cb_w, val, s, w_idx, w_r, fp8=fp8)
    y16 = _offset16(y)
    B.qgemm_values(cb_w, val, s, w_idx, w_r, y=y16, fp8=fp8)
    a_idx, s_c = B.quantize_acts(plan, cb_a, x)
    yc = (B.qgemm_fp8 if fp8 else B.qgemm)(cb_a, cb_w, a_idx, s_c, w_idx, w_r)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert y.data_ptr() % 32 == 0
    assert torch.equal(y16, y)
    assert torch.equal(yc, y)
