"""Pins for the fp64 CPU oracle: each check ties it to something other than
itself (a published table, a closed form, a library routine, brute force or
an exact invariant), so that a dropped term, a wrong sign or index or a
transposed operand anywhere in it fails here.

Method source: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461),
section 方法 (Method).
"""
import os
import math

import numpy as np
import pytest
import scipy.linalg
import scipy.special as sp

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# (d, bits) pairs the five workloads need (activation and weight codebooks)
CONFIG_CODEBOOKS = [(256, 4), (3072, 4), (12288, 4), (4096, 2), (4096, 4), (1536, 4), (1536, 6), (256, 8)]


# --------------------------------------------------------------------------
# independent helpers: the marginal f_d through scipy's regularised
# incomplete beta function (mass) and the closed-form first moment
# --------------------------------------------------------------------------
def log_cd(d):
    """log of c_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) at 40 digits (mpmath)."""
    import mpmath

    with mpmath.workdps(40):
        return float(mpmath.loggamma(mpmath.mpf(d) / 2) - mpmath.log(mpmath.pi) / 2
                     - mpmath.loggamma(mpmath.mpf(d - 1) / 2))


def fd_mass(d, lo, hi):
    """P(lo < T < hi) for T ~ f_d, through the regularised incomplete beta
    function at 40 digits (mpmath): P(|T| < x) = I_{x^2}(1/2, (d-1)/2)."""
    import mpmath

    with mpmath.workdps(40):
        a, b = mpmath.mpf(1) / 2, mpmath.mpf(d - 1) / 2

        def half_mass(x):  # P(0 < T < x) for x >= 0
            x = mpmath.mpf(x)
            return mpmath.betainc(a, b, 0, x * x, regularized=True) / 2

        def signed(x):  # P(0 < T < x) signed
            x = max(-1.0, min(1.0, float(x)))
            return half_mass(x) if x >= 0 else -half_mass(-x)

        return float(signed(hi) - signed(lo))


def fd_first_moment(d, lo, hi):
    """Closed form: int_lo^hi t f_d(t) dt = c_d [(1-lo^2)^((d-1)/2) - (1-hi^2)^((d-1)/2)] / (d-1)."""
    lc = log_cd(d)

    def term(t):
        if abs(t) >= 1.0:
            return 0.0
        return math.exp(lc + 0.5 * (d - 1) * math.log1p(-t * t))

    return (term(lo) - term(hi)) / (d - 1)


def read_golden_max():
    tab = {}
    with open(os.path.join(GOLDEN, "max1960_gaussian_lloyd_max.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            tab.setdefault(int(parts[0]), {})[parts[1]] = [float(v) for v in parts[2:]]
    return tab


# --------------------------------------------------------------------------
# plan
# --------------------------------------------------------------------------
def test_splitmix64_published_vector():
    with open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    seed = int(rows[0][1])
    want = [int(r[0]) for r in rows[1:]]
    got = [int(v) for v in oracle.splitmix64(seed, len(want))]
    assert got == want


@pytest.mark.parametrize("d,h", [(256, 64), (3072, 128), (1536, 128)])
def test_plan_is_a_bijection_with_rademacher_signs(d, h):
    perm, sign = oracle.plan(d, h, 7)
    assert sorted(perm.tolist()) == list(range(d))
    assert set(np.unique(sign).tolist()) <= {-1, 1}
    # a shuffle, not the identity; signs roughly balanced
    assert (perm != np.arange(d)).mean() > 0.9
    assert abs(sign.mean()) < 5.0 / math.sqrt(d)


def _golden_fisher_yates():
    with open(os.path.join(GOLDEN, "fisher_yates_d5_seed1234567.txt")) as f:
        rows = {ln.split()[0]: ln.split()[1:] for ln in f if ln.strip() and not ln.startswith("#")}
    return int(rows["seed"][0]), int(rows["d"][0]), [int(v) for v in rows["perm"]], int(rows["sign0"][0])


def test_plan_shuffle_order_matches_hand_derived_golden():
    """The shuffle's loop direction and swap rule, pinned by a permutation
    derived by hand from the published SplitMix64 outputs (golden file)."""
    seed, d, perm_want, sign0 = _golden_fisher_yates()
    perm, sign = oracle.plan(d, d, seed)
    assert perm.tolist() == perm_want
    assert int(sign[0]) == sign0


def test_plan_permutation_is_uniform():
    """Fisher-Yates over SplitMix64 draws every permutation of 4 items equally often."""
    n = 24000
    counts = {}
    sign_sum = np.zeros(4)
    for seed in range(n):
        perm, sign = oracle.plan(4, 4, seed)
        counts[tuple(perm.tolist())] = counts.get(tuple(perm.tolist()), 0) + 1
        sign_sum += sign
    assert len(counts) == 24
    exp = n / 24.0
    chi2 = sum((c - exp) ** 2 / exp for c in counts.values())
    assert chi2 < 60.0  # 23 dof; p ~ 1e-4 at 54
    assert np.all(np.abs(sign_sum) < 5 * math.sqrt(n))


def test_block_rht_plan_is_identity_with_the_first_draws_as_signs():
    """The ablation plan without P_pi: identity permutation; sign k is the top
    bit of the k-th SplitMix64 output (the generator is pinned above)."""
    d = 256
    perm, sign = oracle.plan(d, 64, 1234567, variant=oracle.BLOCK_RHT)
    np.testing.assert_array_equal(perm, np.arange(d))
    draws = oracle.splitmix64(1234567, d)
    np.testing.assert_array_equal(sign, np.where((draws >> np.uint64(63)) == 1, -1, 1))
    # the RPBH plan of the same seed takes its signs after the d - 1 shuffle draws
    _, sign_rpbh = oracle.plan(d, 64, 1234567)
    draws = oracle.splitmix64(1234567, 2 * d - 1)
    np.testing.assert_array_equal(sign_rpbh, np.where((draws[d - 1:] >> np.uint64(63)) == 1, -1, 1))


def test_plan_rejects_ragged_blocks():
    with pytest.raises(ValueError):
        oracle.plan(100, 64, 0)


# --------------------------------------------------------------------------
# the marginal f_d and its quadrature
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [8, 64, 256, 3072, 12288])
def test_fd_normalised_and_moments_match_closed_forms(d):
    mass, first = oracle.fd_moments(d, -1.0, 1.0)
    assert abs(mass - 1.0) < 1e-13
    assert abs(first) < 1e-15
    for lo, hi in [(0.0, 1.0), (0.5 / math.sqrt(d), 2.0 / math.sqrt(d)), (-3.0 / math.sqrt(d), -0.1 / math.sqrt(d))]:
        m, f1 = oracle.fd_moments(d, lo, hi)
        assert m == pytest.approx(fd_mass(d, lo, hi), rel=1e-12, abs=1e-15)
        assert f1 == pytest.approx(fd_first_moment(d, lo, hi), rel=1e-12, abs=1e-17)


# --------------------------------------------------------------------------
# codebook
# --------------------------------------------------------------------------
@pytest.mark.parametrize("levels", [2, 4, 8, 16])
def test_gaussian_solver_reproduces_max_1960(levels):
    tab = read_golden_max()[levels]
    c, t = oracle.codebook_gauss(levels)
    half = levels // 2
    np.testing.assert_allclose(c[half:], tab["outputs"], atol=2e-3, rtol=0)
    np.testing.assert_allclose(t[half - 1:], tab["thresholds"], atol=2e-3, rtol=0)
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    p = np.diff(sp.ndtr(edges))
    mse = 1.0 - np.sum(p * c * c)  # orthogonality principle at the optimum
    assert mse == pytest.approx(tab["mse"][0], rel=2e-3)


@pytest.mark.parametrize("d,bits", CONFIG_CODEBOOKS)
def test_codebook_satisfies_lloyd_max_conditions(d, bits):
    """Each centroid is the conditional mean of its cell under f_d (scipy's
    incomplete beta for the mass, the closed-form first moment), each
    threshold is the midpoint of its neighbours, the codebook is symmetric."""
    c, t = oracle.codebook(d, bits)
    L = 1 << bits
    sd = math.sqrt(d)
    assert np.all(np.diff(c) > 0)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-15 / sd)
    edges = [-1.0] + list(t) + [1.0]
    for j in range(L):
        m = fd_mass(d, edges[j], edges[j + 1])
        f1 = fd_first_moment(d, edges[j], edges[j + 1])
        assert abs((f1 / m - c[j]) * sd) < 1e-9, (j, f1 / m, c[j])
    if L % 2 == 0:
        assert t[L // 2 - 1] == 0.0


@pytest.mark.parametrize("d,bits", [(256, 4), (1536, 6), (4096, 2)])
def test_raw_solver_is_symmetric(d, bits):
    c, _ = oracle.codebook(d, bits, symmetrize=False)
    assert np.max(np.abs(c + c[::-1])) * math.sqrt(d) < 1e-13


@pytest.mark.parametrize("d", [4, 8, 64, 256, 3072])
def test_one_bit_codebook_closed_form(d):
    """For two levels the centroid is E[T | T > 0] = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))."""
    c, t = oracle.codebook(d, 1)
    want = math.exp(sp.gammaln(d / 2.0) - 0.5 * math.log(math.pi) - sp.gammaln((d + 1) / 2.0))
    assert c[1] == pytest.approx(want, rel=1e-12)
    assert c[0] == -c[1]
    assert t[0] == 0.0


@pytest.mark.parametrize("bits", [2, 4])
def test_codebook_tends_to_the_gaussian_quantiser(bits):
    """sqrt(d) C_d approaches the N(0,1) Lloyd-Max quantiser at rate O(1/d)."""
    cg, _ = oracle.codebook_gauss(1 << bits)
    errs = []
    for d in (768, 3072, 12288):
        c, _ = oracle.codebook(d, bits)
        errs.append(np.max(np.abs(c * math.sqrt(d) - cg)))
    scaled = np.array(errs) * np.array([768, 3072, 12288])
    assert np.all(scaled < 10.0)
    assert np.max(scaled) / np.min(scaled) < 1.02  # error * d is constant: O(1/d)


@pytest.mark.parametrize("d,bits", [(256, 4), (3072, 4), (1536, 6), (4096, 2)])
def test_codebook_orthogonality_principle(d, bits):
    """At a Lloyd-Max optimum E[Q] = 0 and E[T Q(T)] = E[Q(T)^2]; the
    distortion 1/d - E[Q^2] is then close to the Gaussian one divided by d."""
    c, t = oracle.codebook(d, bits)
    L = 1 << bits
    edges = [-1.0] + list(t) + [1.0]
    p = np.array([fd_mass(d, edges[j], edges[j + 1]) for j in range(L)])
    f1 = np.array([fd_first_moment(d, edges[j], edges[j + 1]) for j in range(L)])
    assert abs(np.sum(p * c)) * math.sqrt(d) < 1e-12
    assert np.sum(f1 * c) == pytest.approx(np.sum(p * c * c), rel=1e-10)
    dist = 1.0 / d - np.sum(p * c * c)
    cg, tg = oracle.codebook_gauss(L)
    pg = np.diff(sp.ndtr(np.concatenate([[-np.inf], tg, [np.inf]])))
    dg = 1.0 - np.sum(pg * cg * cg)
    assert dist * d == pytest.approx(dg, rel=2e-2)


# --------------------------------------------------------------------------
# RPBH rotation
# --------------------------------------------------------------------------
def dense_rpbh(d, h, perm, sign):
    """Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi built with scipy's Sylvester Hadamard."""
    H = scipy.linalg.hadamard(h).astype(np.float64) / math.sqrt(h)
    blocks = [H @ np.diag(sign[b * h:(b + 1) * h].astype(np.float64)) for b in range(d // h)]
    B = scipy.linalg.block_diag(*blocks)
    P = np.zeros((d, d))
    P[np.arange(d), perm] = 1.0  # (P x)_k = x[perm[k]]
    return B @ P


@pytest.mark.parametrize("d,h,seed", [(256, 64, 0), (512, 128, 3), (384, 128, 11)])
def test_rpbh_matches_dense_definition(d, h, seed):
    perm, sign = oracle.plan(d, h, seed)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((5, d))
    y = oracle.rpbh(x, h, perm, sign)
    want = x @ dense_rpbh(d, h, perm, sign).T
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-13)


def test_rpbh_identity_plan_is_block_hadamard():
    d, h = 256, 64
    perm = np.arange(d, dtype=np.int32)
    sign = np.ones(d, dtype=np.int8)
    x = np.random.default_rng(1).standard_normal((3, d))
    H = scipy.linalg.hadamard(h) / math.sqrt(h)
    want = np.concatenate([x[:, b * h:(b + 1) * h] @ H.T for b in range(d // h)], axis=1)
    np.testing.assert_allclose(oracle.rpbh(x, h, perm, sign), want, atol=1e-13, rtol=0)


def test_rpbh_is_orthogonal():
    d, h = 256, 64
    perm, sign = oracle.plan(d, h, 0)
    Pi = oracle.rpbh(np.eye(d), h, perm, sign).T  # column k = Pi e_k
    assert np.max(np.abs(Pi @ Pi.T - np.eye(d))) < 1e-14
    x = np.random.default_rng(2).standard_normal((4, d)) * 3.0
    y = oracle.rpbh(x, h, perm, sign)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)


def test_rotation_cancels_in_the_product():
    """(W Pi^T)(Pi x) = W x: the weight side absorbs Pi^T (row n of W' is Pi w_n)."""
    d, h, N = 512, 128, 40
    perm, sign = oracle.plan(d, h, 5)
    rng = np.random.default_rng(5)
    W = rng.standard_normal((N, d)) * 0.02
    x = rng.standard_normal((7, d))
    Wp = oracle.rpbh(W, h, perm, sign)
    xp = oracle.rpbh(x, h, perm, sign)
    got = xp @ Wp.T
    want = x @ W.T
    assert np.linalg.norm(got - want) / np.linalg.norm(want) < 1e-12


def _outlier_unit_vector(d, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(d)
    x[rng.choice(d, 4, replace=False)] *= 20.0
    return x / np.linalg.norm(x)


def test_permutation_makes_every_coordinate_variance_one_over_d():
    """Over random (pi, signs), E[(Pi x~)_k^2] = 1/d exactly for every unit x~;
    without the permutation (Block-RHT) the blocks holding outlier channels
    carry far more than 1/d."""
    d, h, n = 256, 64, 1000
    x = _outlier_unit_vector(d, 100)[None, :]
    ys = np.empty((n, d))
    yb = np.empty((n, d))
    ident = np.arange(d, dtype=np.int32)
    for seed in range(n):
        perm, sign = oracle.plan(d, h, 10_000 + seed)
        ys[seed] = oracle.rpbh(x, h, perm, sign)[0]
        yb[seed] = oracle.rpbh(x, h, ident, sign)[0]

    def zscores(y):
        sq = y * y
        se = sq.std(axis=0, ddof=1) / math.sqrt(n)
        return (sq.mean(axis=0) - 1.0 / d) / se

    z = zscores(ys)
    assert np.mean(z * z) < 2.0 and np.max(np.abs(z)) < 5.5
    assert np.max(np.abs(zscores(yb))) > 20.0


# --------------------------------------------------------------------------
# quantiser
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d,bits", [(64, 2), (64, 4), (64, 6), (256, 8)])
def test_threshold_count_is_the_nearest_centroid(d, bits):
    """Brute force on 1e5 coordinates of random unit directions."""
    h = 64
    c, t = oracle.codebook(d, bits)
    perm, sign = oracle.plan(d, h, 1)
    x = np.random.default_rng(bits).standard_normal((100_032 // d, d))
    out = oracle.quantize_rows(x, h, perm, sign, t, decision=64, want_v=True)
    v = out["v"]
    brute = np.argmin(np.abs(v[..., None] - c[None, None, :]), axis=-1)
    assert np.array_equal(out["idx"], brute.astype(np.uint8))
    np.testing.assert_allclose(np.linalg.norm(v, axis=1), 1.0, rtol=1e-12)


def test_quantiser_norm_and_direction_split():
    d, h = 256, 64
    c, t = oracle.codebook(d, 4)
    perm, sign = oracle.plan(d, h, 0)
    x = np.random.default_rng(9).standard_normal((4, d)) * np.array([[1.0], [5.0], [0.01], [300.0]])
    out = oracle.quantize_rows(x, h, perm, sign, t, decision=64, want_y=True, want_v=True)
    np.testing.assert_allclose(out["s"], np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(out["v"] * (out["s"][:, None] + oracle.EPS), out["y"], rtol=1e-13, atol=0)
    # the direction, not the scale, decides the index
    assert np.array_equal(out["idx"][0], oracle.quantize_rows(x[:1] * 7.0, h, perm, sign, t, decision=64)["idx"][0])


def test_zero_row_takes_the_upper_middle_cell():
    """v = 0 sits on the middle threshold t = 0; ties go to the upper cell."""
    d, h = 256, 64
    for bits in (2, 4, 6):
        c, t = oracle.codebook(d, bits)
        perm, sign = oracle.plan(d, h, 0)
        out = oracle.quantize_rows(np.zeros((2, d)), h, perm, sign, t, decision=32)
        assert np.all(out["idx"] == (1 << bits) // 2)
        assert np.all(out["s"] == 0.0)


def test_fp32_decision_differs_only_next_to_thresholds():
    d, h = 3072, 128
    c, t = oracle.codebook(d, 4)
    perm, sign = oracle.plan(d, h, 1)
    x = np.random.default_rng(3).standard_normal((16, d))
    a = oracle.quantize_rows(x, h, perm, sign, t, decision=64, want_v=True)
    b = oracle.quantize_rows(x, h, perm, sign, t, decision=32)
    diff = a["idx"] != b["idx"]
    if diff.any():
        v = a["v"][diff]
        dist = np.min(np.abs(v[:, None] - t[None, :]), axis=1)
        assert np.all(dist <= 1e-6 * np.maximum(np.abs(v), 1 / math.sqrt(d)))


# --------------------------------------------------------------------------
# bf16 rounding and the quantised product
# --------------------------------------------------------------------------
def test_bf16_rounding_matches_torch():
    import torch

    rng = np.random.default_rng(4)
    vals = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-8, 8, 10000),
                           [0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3.0e38]])
    vals = vals.astype(np.float32).astype(np.float64)  # fp32 inputs: one rounding either way
    bits, val = oracle.round_bf16(vals)
    tb = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)
    np.testing.assert_array_equal(bits, tb.view(torch.int16).numpy().view(np.uint16))
    np.testing.assert_array_equal(val, tb.to(torch.float64).numpy())


def test_bf16_rounding_of_fp64_is_a_single_rounding():
    """A value just above a bf16 midpoint whose fp32 image lands on the
    midpoint: one rounding from fp64 goes up, fp32-then-bf16 would tie to even."""
    x = 1.0 + 2 ** -8 + 2 ** -40
    bits, val = oracle.round_bf16(np.array([x]))
    assert val[0] == 1.0 + 2 ** -7
    # the exact bf16 neighbours bracket x; the nearer one wins
    lo, hi = 1.0, 1.0 + 2 ** -7
    assert abs(val[0] - x) <= min(abs(lo - x), abs(hi - x))


def test_qlinear_reduces_to_an_integer_matmul():
    """With integer-valued stand-in centroids the product is an exact integer
    GEMM scaled by r[n] and s[m] on the output's columns and rows."""
    rng = np.random.default_rng(6)
    M, N, d, L = 37, 23, 96, 16
    ia = rng.integers(0, L, (M, d)).astype(np.uint8)
    iw = rng.integers(0, L, (N, d)).astype(np.uint8)
    ca = np.arange(L, dtype=np.float64) - 7.0
    cw = 3.0 - np.arange(L, dtype=np.float64) * 2.0
    s = rng.uniform(0.5, 2.0, M)
    r = rng.uniform(0.5, 2.0, N)
    got = oracle.qlinear(ia, s, iw, r, ca, cw)
    want = (ca[ia] @ cw[iw].T) * s[:, None] * r[None, :]
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=0)
    rows = np.array([36, 0, 5])
    cols = np.array([22, 1])
    np.testing.assert_allclose(oracle.qlinear(ia, s, iw, r, ca, cw, rows, cols), want[rows][:, cols], rtol=1e-15)


def test_quantised_product_error_falls_with_bits():
    """End to end (x, W) -> y through the oracle: the relative error of the
    quantised product against x W^T shrinks as bits grow, at the size the
    per-coordinate distortion predicts."""
    d, h, M, N = 256, 64, 64, 256
    rng = np.random.default_rng(100)
    x = rng.standard_normal((M, d))
    x[:, rng.choice(d, 4, replace=False)] *= 20.0
    W = rng.standard_normal((N, d)) * 0.02
    perm, sign = oracle.plan(d, h, 0)
    ref = x @ W.T
    errs = []
    for bits in (2, 4, 6):
        c, t = oracle.codebook(d, bits)
        qa = oracle.quantize_rows(x, h, perm, sign, t, decision=64)
        qw = oracle.quantize_rows(W, h, perm, sign, t, decision=64)
        y = oracle.qlinear(qa["idx"], qa["s"], qw["idx"], qw["s"], c, c)
        errs.append(np.linalg.norm(y - ref) / np.linalg.norm(ref))
    assert errs[0] > errs[1] > errs[2]
    assert errs[1] < 0.2 and errs[2] < 0.06


@pytest.mark.parametrize("d", [1536, 3072, 4096, 12288])
def test_stored_eight_bit_codebooks_satisfy_lloyd_max_conditions(d):
    """The oracle's stored 8-bit codebooks (tests/golden, written by
    make_oracle_codebooks.py from oracle.codebook) are pinned the same way
    as the solved ones: ascending, antisymmetric, thresholds at midpoints,
    each centroid the conditional mean of its cell under f_d (scipy's
    incomplete beta for the mass, the closed-form first moment)."""
    from stored_codebooks import stored_oracle_codebook

    c, t = stored_oracle_codebook(d, 8)
    L = 256
    sd = math.sqrt(d)
    assert c.shape == (L,) and t.shape == (L - 1,)
    assert np.all(np.diff(c) > 0)
    np.testing.assert_array_equal(c, -c[::-1])
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-15 / sd)
    assert t[L // 2 - 1] == 0.0
    edges = [-1.0] + list(t) + [1.0]
    for j in range(0, L, 5):
        m = fd_mass(d, edges[j], edges[j + 1])
        f1 = fd_first_moment(d, edges[j], edges[j + 1])
        assert abs((f1 / m - c[j]) * sd) < 1e-9, (j, f1 / m, c[j])
