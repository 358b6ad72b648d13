"""Seeded synthetic inputs for the five workload shapes.

This module holds the input recipes only (value distributions, shapes,
seeds); none of the method's arithmetic lives here.  The GPU path and the
fp64 oracle both read their inputs from it, so that both see the same bytes.

The shapes stand in for FLUX.1-, 7B single-stream-DiT- and Wan-style linear
layers (the workloads the OrbitQuant page evaluates on); no model weights,
prompts or datasets are used.
"""
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    M: int  # tokens
    d: int  # input dim (= K of the GEMM)
    N: int  # output dim
    h: int  # RPBH block size
    bits_w: int
    bits_a: int
    x_dtype: str  # "f32" or "bf16"
    plan_seed: int
    data_seed: int
    x_recipe: str
    w_recipe: str

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.d


WORKLOADS = {
    "tiny_w4a4": Workload("tiny_w4a4", 64, 256, 256, 64, 4, 4, "f32", 0, 100,
                          "normal_outlier4x20", "normal0.02"),
    "flux_qkv_w4a4": Workload("flux_qkv_w4a4", 4096, 3072, 9216, 128, 4, 4, "bf16", 1, 101,
                              "student_t3_lognorm1", "normal0.02_rows1pct_x8"),
    "flux_mlp_down_w4a4": Workload("flux_mlp_down_w4a4", 4096, 12288, 3072, 128, 4, 4, "bf16", 2, 102,
                                   "gelu_lognorm1.5", "normal0.01"),
    "dit7b_mlp_up_w2a4": Workload("dit7b_mlp_up_w2a4", 16384, 4096, 16384, 128, 2, 4, "bf16", 3, 103,
                                  "student_t2.5_lognorm1", "normal0.015"),
    "video_ffn_w4a6": Workload("video_ffn_w4a6", 32760, 1536, 8960, 128, 4, 6, "bf16", 4, 104,
                               "normal_lognorm1_spikes0.1pct_x50", "normal0.02"),
}
ORDER = ["tiny_w4a4", "flux_qkv_w4a4", "flux_mlp_down_w4a4", "dit7b_mlp_up_w2a4", "video_ffn_w4a6"]


def _to_dtype(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t if dtype == "f32" else t.to(torch.bfloat16)


def _gelu(z: np.ndarray) -> np.ndarray:
    # exact (erf) GELU of the pre-activation; part of the input recipe
    from scipy.special import erf

    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def make_x(w: Workload, rows=None, M=None) -> torch.Tensor:
    """Activations [M, d] in the workload's dtype (CPU tensor).  The
    per-channel scales depend only on the seed, so a row subset (``rows``) is
    the same data as the full tensor's rows."""
    M = w.M if M is None else M
    rng = np.random.default_rng(w.data_seed)
    d = w.d
    r = w.x_recipe
    # per-channel structure first (independent of M)
    if r == "normal_outlier4x20":
        chan = np.ones(d)
        chan[rng.choice(d, 4, replace=False)] = 20.0
    elif r.startswith("student_t3") or r.startswith("student_t2.5") or r.startswith("normal_lognorm1"):
        chan = np.exp(rng.normal(0.0, 1.0, d))
    elif r == "gelu_lognorm1.5":
        chan = np.exp(rng.normal(0.0, 1.5, d))
    else:
        raise ValueError(r)
    spikes = None
    if r == "normal_lognorm1_spikes0.1pct_x50":
        n_sp = max(1, int(round(M * 0.001)))
        spikes = rng.choice(M, n_sp, replace=False)
    idx = np.arange(M) if rows is None else np.asarray(rows)
    out = np.empty((len(idx), d), dtype=np.float32)
    # per-row values from a row-keyed stream so that subsets match the whole
    chunk = 1024
    for c0 in range(0, len(idx), chunk):
        sel = idx[c0:c0 + chunk]
        vals = np.empty((len(sel), d), dtype=np.float64)
        for j, m in enumerate(sel):
            g = np.random.default_rng([w.data_seed, 1, int(m)])
            if r == "normal_outlier4x20":
                vals[j] = g.standard_normal(d)
            elif r.startswith("student_t3"):
                vals[j] = g.standard_t(3.0, d)
            elif r.startswith("student_t2.5"):
                vals[j] = g.standard_t(2.5, d)
            elif r == "gelu_lognorm1.5":
                vals[j] = _gelu(g.standard_normal(d))
            else:
                vals[j] = g.standard_normal(d)
        vals *= chan[None, :]
        if spikes is not None:
            hit = np.isin(sel, spikes)
            vals[hit] *= 50.0
        out[c0:c0 + len(sel)] = vals
    return _to_dtype(out, w.x_dtype)


def make_w(w: Workload, rows=None) -> torch.Tensor:
    """Weights [N, d] (fp32 for the tiny case, bf16 otherwise; CPU tensor)."""
    rng = np.random.default_rng([w.data_seed, 2])
    N, d = w.N, w.d
    r = w.w_recipe
    std = float(r.split("_")[0].replace("normal", ""))
    big = None
    if r.endswith("rows1pct_x8"):
        big = rng.choice(N, max(1, int(round(N * 0.01))), replace=False)
    W = rng.standard_normal((N, d), dtype=np.float32) * np.float32(std)
    if big is not None:
        W[big] *= np.float32(8.0)
    if rows is not None:
        W = W[np.asarray(rows)]
    return _to_dtype(W, w.x_dtype)


def recipe_text(w: Workload) -> str:
    return (f"{w.name}: M={w.M} d={w.d} N={w.N} h={w.h} W{w.bits_w}A{w.bits_a} x:{w.x_recipe} ({w.x_dtype}) "
            f"W:{w.w_recipe} plan_seed={w.plan_seed} data_seed={w.data_seed}")
