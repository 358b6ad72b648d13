"""Shared parity machinery: run the CUDA path through the C ABI and compare it
with the fp64 oracle on the same seeded inputs.

Tolerances (stated here, used by every parity test):
  - indices: bit-exact, except coordinates whose oracle direction v lies
    within 1e-6 * max(|t_j|, 1/sqrt(d)) of a decision threshold t_j; those
    are counted and must stay below 1e-5 of the checked coordinates;
  - rotated values: |dy| <= 1e-5 (|y_k| + s/sqrt(d)); norms s: 1e-5 relative;
  - stored bf16 row norms: equal, or one bf16 ulp apart when the fp32 norm
    sits next to a rounding midpoint (counted);
  - quantised product: relative Frobenius error <= 2e-3 against the oracle's
    fp64 product of the same indices, norms and bf16 centroid values, and
    element by element |y - ref| <= 2^-8 |ref| + 2^-8 rms(ref): half a bf16
    ulp of the output (2^-8 relative) plus the same fraction of the
    product's rms for the fp32 accumulation's rounding near zero.  No element
    may exceed it.
"""
import math

import numpy as np
import torch

import oracle
from rotation_bit_quantization_rpbh_b200 import binding as B
from stored_codebooks import stored_oracle_codebook  # noqa: F401  (re-exported for the parity tests)

BAND_REL = 1e-6
MISMATCH_FRAC = 1e-5
ROT_TOL = 1e-5
GEMM_TOL = 2e-3
ELEM_REL = 2.0 ** -8


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a CPU bf16/fp32 tensor to fp64."""
    return t.detach().cpu().to(torch.float32).numpy().astype(np.float64)


def check_indices(gpu_idx, or_idx, v64, t64, d, total=None):
    """Returns the number of in-band mismatches; asserts every mismatch is in
    band and that they are fewer than 1e-5 of `total` coordinates (default:
    the coordinates given)."""
    mis = gpu_idx != or_idx
    n = int(mis.sum())
    if n == 0:
        return 0
    vv = v64[mis]
    j = np.argmin(np.abs(vv[:, None] - t64[None, :]), axis=1)
    dist = np.abs(vv - t64[j])
    band = BAND_REL * np.maximum(np.abs(t64[j]), 1.0 / math.sqrt(d))
    assert np.all(dist <= band), f"{int(np.sum(dist > band))} index mismatches outside the threshold band"
    total = gpu_idx.size if total is None else total
    assert n < MISMATCH_FRAC * total, f"{n} in-band mismatches of {total}"
    return n


def check_rotation(plan, X_cpu, rows, h, perm, sign, dev):
    xg = X_cpu.to(dev)
    y, nrm = B.rpbh_apply(plan, xg)
    torch.cuda.synchronize()
    y = y.cpu().numpy().astype(np.float64)[rows]
    nrm = nrm.cpu().numpy().astype(np.float64)[rows]
    x64 = to_f64(X_cpu[rows])
    y_or = oracle.rpbh(x64, h, perm, sign)
    s_or = np.linalg.norm(y_or, axis=1)
    d = X_cpu.shape[1]
    tol = ROT_TOL * (np.abs(y_or) + s_or[:, None] / math.sqrt(d))
    assert np.all(np.abs(y - y_or) <= tol), float(np.max(np.abs(y - y_or) / tol))
    np.testing.assert_allclose(nrm, s_or, rtol=ROT_TOL, atol=0)


def check_quantized_rows(idx_gpu_packed, scale_gpu, X_cpu, rows, h, perm, sign, cb, oracle_cb, kind, chunk=2048):
    """kind 'acts': scale is s (fp32); 'weights': scale is r (bf16).  Rows are
    checked in chunks (the oracle's fp64 copy of a full-size input would not
    fit comfortably); the oracle's v is recomputed only for rows with a
    mismatch.  Returns (in-band mismatches, one-ulp norm differences)."""
    d = X_cpu.shape[1]
    c64, t64 = oracle_cb
    rows = np.asarray(rows)
    n_band = n_ulp = 0
    for i0 in range(0, len(rows), chunk):
        rr = rows[i0:i0 + chunk]
        gi = B.unpack_indices(idx_gpu_packed[torch.as_tensor(rr, device=idx_gpu_packed.device)], d, cb.bits)
        gi = gi.cpu().numpy()
        x64 = to_f64(X_cpu[rr])
        out = oracle.quantize_rows(x64, h, perm, sign, t64, decision=32)
        bad = np.where((gi != out["idx"]).any(axis=1))[0]
        if len(bad):
            ov = oracle.quantize_rows(x64[bad], h, perm, sign, t64, decision=32, want_v=True)
            n_band += check_indices(gi[bad], ov["idx"], ov["v"], t64, d, total=len(rows) * d)
        sc = scale_gpu[torch.as_tensor(rr, device=scale_gpu.device)].cpu()
        if kind == "acts":
            np.testing.assert_allclose(sc.numpy().astype(np.float64), out["s"], rtol=ROT_TOL, atol=0)
        else:
            got = sc.view(torch.int16).numpy().astype(np.int64) & 0xFFFF
            want = oracle.round_bf16(out["s"])[0].astype(np.int64)
            diff = np.abs(got - want)
            assert np.all(diff <= 1), "stored row norms differ by more than one bf16 ulp"
            n_ulp += int(np.sum(diff == 1))
            # a one-ulp difference only where the fp32 norm is next to a bf16 midpoint
            if np.any(diff == 1):
                r64 = out["s"][diff == 1]
                lo = oracle.round_bf16(r64 * (1 - 2e-6))[1]
                hi = oracle.round_bf16(r64 * (1 + 2e-6))[1]
                assert np.all(lo != hi)
    assert n_band < MISMATCH_FRAC * len(rows) * d, f"{n_band} in-band mismatches of {len(rows) * d}"
    return n_band, n_ulp


def check_product(y_gpu64, ref):
    """Relative Frobenius error <= GEMM_TOL and the element-wise bound (see
    the module docstring).  Returns (relative error, elements over the bound,
    worst |y - ref| / bound)."""
    err = rel_frob(y_gpu64, ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = ELEM_REL * np.abs(ref) + ELEM_REL * rms
    over = np.abs(y_gpu64 - ref) > bound
    n_over = int(over.sum())
    worst = float(np.max(np.abs(y_gpu64 - ref) / np.maximum(bound, 1e-300))) if ref.size else 0.0
    assert err <= GEMM_TOL, err
    assert n_over == 0, f"{n_over} product elements outside |y - ref| <= 2^-8 |ref| + 2^-8 rms (worst {worst:.2f}x)"
    return err, n_over, worst


def gemm_reference(ia_full, s, iw_full, r, ca, cw, rows=None, cols=None):
    return oracle.qlinear(ia_full, s, iw_full, r, ca, cw, rows, cols)


def rel_frob(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
