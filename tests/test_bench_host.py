"""Host-side helpers of bench.py (no GPU): the Full RHT block reading, the
steady-state fit of the quantiser sweep, the kernel-source digest that keys
the committed traffic figures, and the whole-job throughput."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("d,h", [(3072, 1024), (12288, 4096), (4096, 4096), (1536, 512), (256, 256),
                                 (16384, 16384), (32768, 16384), (96, 32)])
def test_full_rht_block_is_the_largest_power_of_two_dividing_d(d, h):
    """Full RHT takes one Sylvester block over d where d is a power of two,
    else the largest power-of-two block dividing d (capped at the staged
    kernel's 16384)."""
    assert bench.full_rht_block(d) == h
    assert d % h == 0 and h & (h - 1) == 0


def test_steady_fit_recovers_a_linear_cost():
    """A line through (M, us) with a known per-row cost and intercept gives
    them back, and the rate is bytes per row over the per-row time."""
    per_row, peak = 7684, 6548.2
    rows = [{"M": M, "codes_us": 8.0 + 0.003 * M} for M in (4096, 8192, 16384, 32768)]
    f = bench.steady_fit(rows, per_row, peak, 8192)
    assert f["fit_M"] == [8192, 16384, 32768]
    assert f["us_per_row"] == pytest.approx(0.003, rel=1e-9)
    assert f["intercept_us"] == pytest.approx(8.0, rel=1e-9)
    gbs = per_row / (0.003e-6) / 1e9
    assert f["steady_gbs"] == pytest.approx(gbs, rel=1e-9)
    assert f["steady_frac"] == pytest.approx(gbs / peak, rel=1e-9)
    assert bench.steady_fit(rows, per_row, peak, 32768) is None  # one point is no line


def test_code_digest_ignores_comments_but_not_code():
    a = "// a comment\nint f(int x) {  /* inline */ return x + 1; }\n\n#include <x.h>\n"
    b = "int f(int x) { return x + 1; }  // another comment\n"
    c = "int f(int x) { return x + 2; }\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(c)


def test_every_traffic_entry_names_a_known_kernel():
    """profiles/traffic.json keys are kernels bench.py reports, each with a
    digest of the sources it is computed from."""
    import json

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    for k, v in t.items():
        if k.startswith("_"):
            continue
        assert k in bench.KERNEL_SOURCES, k
        assert len(v["code_md5"]) == 32
        assert all(isinstance(n, int) and n > 0 for key, n in v.items() if key != "code_md5")
    assert len(bench.kernel_code_md5("rpbh_quant")) == 32


def test_job_throughput_is_all_ranks_tokens_over_the_step():
    assert bench.job_throughput(1, 4096, 0.25) == pytest.approx(4096 / 0.25e-3)
    assert bench.job_throughput(8, 4096, 0.25) == pytest.approx(8 * 4096 / 0.25e-3)
    assert np.isfinite(bench.job_throughput(2, 1, 1.0))
