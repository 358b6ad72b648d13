"""fp64 CPU oracle for the OrbitQuant rotate-then-quantize linear layer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg are its only callers.  Nothing in the product
package imports it, and it imports nothing from the product package.

Every function follows the "OrbitQuant" paper summary (hyper.ai, papers
2607.02461), section 方法 (Method); the C source states each step and each
reading taken where the page is silent.  Parity status: every function here
is pinned by tests/test_oracle_pins.py against closed forms, published
tables, library routines or brute force.  The one part left unpinned is the
absolute quality of C_d against the paper's own codebooks, which the page
does not print.

Inputs are plain numpy arrays; bf16 inputs are widened to fp64 exactly by
the caller (see ``widen_bf16``).
"""
import ctypes
import os

import numpy as np

from . import build as _build  # noqa: E402

_lib = None
EPS = 1e-12


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oracle_codebook.argtypes = [ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_codebook_ex.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_codebook_gauss.argtypes = [ctypes.c_int, P, P]
        L.oracle_fd_moments.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double, P, P]
        L.oracle_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_int, P]
        L.oracle_plan.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, P, P]
        L.oracle_plan_variant.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int, P, P]
        L.oracle_rpbh.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.oracle_quantize_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, ctypes.c_int, P,
                                           ctypes.c_double, ctypes.c_int, P, P, P, P]
        L.oracle_round_bf16.argtypes = [ctypes.c_int, P, P, P]
        L.oracle_qlinear.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, ctypes.c_int, P,
                                     ctypes.c_int, P, P]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


_cb_cache = {}


def codebook(d, bits, symmetrize=True):
    """Lloyd-Max codebook C_d for 2**bits levels: (centroids[L], thresholds[L-1]), t units."""
    key = (d, bits, bool(symmetrize))
    if key not in _cb_cache:
        L = 1 << bits
        c = np.zeros(L)
        t = np.zeros(max(L - 1, 1))
        it = lib().oracle_codebook_ex(d, bits, int(bool(symmetrize)), _p(c), _p(t))
        if it < 0:
            raise RuntimeError("oracle codebook did not converge (d=%d bits=%d): %d" % (d, bits, it))
        _cb_cache[key] = (c, t[: L - 1].copy())
    c, t = _cb_cache[key]
    return c.copy(), t.copy()


def codebook_gauss(levels):
    """The same Lloyd-Max solver on N(0, 1) (to pin it against published tables)."""
    c = np.zeros(levels)
    t = np.zeros(levels)
    it = lib().oracle_codebook_gauss(levels, _p(c), _p(t))
    if it < 0:
        raise RuntimeError("no convergence")
    return c, t[: levels - 1].copy()


def fd_moments(d, a, b):
    m0 = np.zeros(1)
    m1 = np.zeros(1)
    lib().oracle_fd_moments(d, float(a), float(b), _p(m0), _p(m1))
    return float(m0[0]), float(m1[0])


def splitmix64(seed, n):
    out = np.zeros(n, dtype=np.uint64)
    lib().oracle_splitmix64(ctypes.c_uint64(seed), n, _p(out))
    return out


BLOCK_RHT = 1  # plan variant without the permutation (the page's rotation ablation)


def plan(d, h, seed, variant=0):
    """RPBH plan (variant 0) or Block-RHT plan (variant 1, identity permutation):
    (perm[d] int32 with (P_pi x)_k = x[perm[k]], sign[d] int8 in {-1,+1})."""
    perm = np.zeros(d, dtype=np.int32)
    sign = np.zeros(d, dtype=np.int8)
    rc = lib().oracle_plan_variant(d, h, ctypes.c_uint64(seed), variant, _p(perm), _p(sign))
    if rc != 0:
        raise ValueError("bad plan arguments")
    return perm, sign


def rpbh(x, h, perm, sign):
    """y = Pi_d x for every row of x (fp64, direct O(h) sums)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    M, d = x.shape
    y = np.zeros_like(x)
    lib().oracle_rpbh(M, d, h, _p(perm), _p(sign), _p(x), _p(y))
    return y


def quantize_rows(x, h, perm, sign, thresholds, decision=32, want_y=False, want_v=False):
    """Rotate, split, quantise rows.  Returns dict(idx uint8 [M,d], s [M], y?, v?)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    M, d = x.shape
    L = len(thresholds) + 1
    thr = np.ascontiguousarray(thresholds, dtype=np.float64)
    idx = np.zeros((M, d), dtype=np.uint8)
    s = np.zeros(M)
    y = np.zeros((M, d)) if want_y else None
    v = np.zeros((M, d)) if want_v else None
    lib().oracle_quantize_rows(M, d, h, _p(perm), _p(sign), _p(x), L, _p(thr), EPS, int(decision), _p(idx), _p(s),
                               _p(y), _p(v))
    out = {"idx": idx, "s": s}
    if want_y:
        out["y"] = y
    if want_v:
        out["v"] = v
    return out


def round_bf16(a):
    """(bits uint16, values fp64) of bf16 round-to-nearest-even of a (through fp32)."""
    a = np.ascontiguousarray(a, dtype=np.float64).ravel()
    bits = np.zeros(a.size, dtype=np.uint16)
    val = np.zeros(a.size)
    lib().oracle_round_bf16(a.size, _p(a), _p(bits), _p(val))
    return bits, val


def qlinear(ia, s, iw, r, ca, cw, rows=None, cols=None):
    """y[m,n] = r[n] s[m] sum_k cw[iw[n,k]] ca[ia[m,k]] (fp64) on the listed rows/cols."""
    ia = np.ascontiguousarray(ia, dtype=np.uint8)
    iw = np.ascontiguousarray(iw, dtype=np.uint8)
    M, d = ia.shape
    N = iw.shape[0]
    s = np.ascontiguousarray(s, dtype=np.float64)
    r = np.ascontiguousarray(r, dtype=np.float64)
    ca = np.ascontiguousarray(ca, dtype=np.float64)
    cw = np.ascontiguousarray(cw, dtype=np.float64)
    rr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    cc = None if cols is None else np.ascontiguousarray(cols, dtype=np.int32)
    nr = M if rr is None else len(rr)
    nc = N if cc is None else len(cc)
    out = np.zeros((nr, nc))
    lib().oracle_qlinear(M, N, d, _p(ia), _p(s), _p(iw), _p(r), _p(ca), _p(cw), nr, _p(rr), nc, _p(cc), _p(out))
    return out


def num_threads():
    return lib().oracle_num_threads()


def set_num_threads(n):
    """Threads of the oracle's parallel loops (n <= 0: the default)."""
    lib().oracle_set_num_threads(int(n))


def widen_bf16(bits_u16):
    """Exact bf16 -> fp64 widening of raw bf16 bit patterns (argument marshalling)."""
    b = np.ascontiguousarray(bits_u16, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
