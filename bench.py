#!/usr/bin/env python
"""Benchmark of the OrbitQuant rotate-then-quantize linear layer on B200.

One step = the whole per-token hot path over one batch: the fused RPBH
rotate + norm split + Lloyd-Max quantise kernel on the activations, then the
codebook-decode tcgen05 GEMM (weights were quantised offline, before timing).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle as the reference arm

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
M tokens against a replicated packed weight -- the path has no exchange, so
there is no data-path collective (weak scaling); only the timing is reduced
(max over ranks).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "qlinear tokens/s and TFLOP/s (% bf16 peak); RPBH+quant GB/s (% HBM peak)"
DEFAULT_WORKLOAD = "flux_qkv_w4a4"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip timing the other large workloads (the per_workload block)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline sample")
    ap.add_argument("--fp8", action="store_true",
                    help="time the fp8 variant of the product (oq_qgemm_fp8: e4m3 centroid values)")
    ap.add_argument("--schedule", default="auto", choices=["auto", "codes", "values"],
                    help="layer schedule timed: activation codes decoded in the GEMM, or centroid values written by "
                         "the quantiser and streamed into the GEMM; auto = the one oq_qlinear takes")
    ap.add_argument("--ablation", action="store_true",
                    help="time the rotation ablation (RPBH, Block-RHT, Full RHT, dense Haar) on --workload instead "
                         "of the layer")
    ap.add_argument("--gemm-sweep", action="store_true",
                    help="time the A-values product alone over a range of M at --workload's d, N and bits (per-round "
                         "rate against the fixed cost) instead of the layer")
    ap.add_argument("--quant-sweep", action="store_true",
                    help="time the quantiser alone over a range of M at --workload's d (fixed cost against per-row "
                         "cost) instead of the layer")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


_RPBH_SOURCES = ("rpbh_quant.cu", "rpbh_groups.cu")  # the team and the warp-group kernel (and their shared epilogue)
KERNEL_SOURCES = {"qgemm": ("qgemm.cu",), "qgemm_fp8": ("qgemm.cu",), "qgemm_values": ("qgemm.cu",),
                  "qgemm_values_fp8": ("qgemm.cu",), "rpbh_quant": _RPBH_SOURCES, "rpbh_quant_values": _RPBH_SOURCES,
                  "rpbh_quant_values_fp8": _RPBH_SOURCES}


def kernel_code_md5(kernel):
    """md5 of the kernel's sources (code_only, concatenated in order)."""
    import hashlib

    parts = []
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "rotation_bit_quantization_rpbh_b200", "csrc", name), encoding="utf-8") as f:
            parts.append(code_only(f.read()))
    return hashlib.md5("\n".join(parts).encode()).hexdigest()


def committed_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if one exists for
    this kernel and workload and the kernel source is unchanged since the
    counters were taken (null otherwise)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f).get(kernel, {})
    if kernel_code_md5(kernel) != j.get("code_md5"):
        return None
    return j.get(workload)


def code_only(src):
    """C++ source with comments, #include lines and blank lines removed and
    whitespace runs collapsed: its digest changes with the code, not with
    its comments."""
    import re

    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    lines = [" ".join(ln.split()) for ln in src.splitlines()]
    return "\n".join(ln for ln in lines if ln and not ln.startswith("#include"))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed loop runs."""

    FIELDS = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.rows = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10:
                self.rows.append((time.time(), parts))

    def mark(self, which):
        if which == "start":
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        mine = [p for (t, p) in self.rows if (not self.uuid or self.uuid in p[1])]
        inside = [p for (t, p) in self.rows if self.t0 and self.t0 - 0.05 <= t <= self.t1 + 0.05 and
                  (not self.uuid or self.uuid in p[1])]
        use = inside if inside else mine[-5:]
        if not use:
            return None
        sm = [float(p[2]) for p in use if p[2].replace(".", "").isdigit()]
        mx = [float(p[3]) for p in use if p[3].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in use:
            for n, v in zip(names, p[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(use), "samples_in_timed_region": len(inside)}


def reduce_max(values, world, device):
    """Element-wise max over ranks of per-rank device times (the slowest rank
    sets the job's time); identity on one rank."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, tokens_per_rank, ms_per_step):
    """Whole-job tokens/s: every rank runs its own batch (weak scaling)."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def rpbh_bytes(w):
    """Algorithmic bytes of one quantiser launch as the method defines its
    output: x read, the packed codes written (one byte per code at 6 bits),
    and s.  The values schedule's 2-byte centroid values are the library's
    layout for the product, not the method's output, so they count in the
    measured traffic only."""
    esize = 4 if w.x_dtype == "f32" else 2
    out = w.d if w.bits_a in (6, 8) else w.d * w.bits_a // 8
    return w.M * (w.d * esize + out + 4)


def cpu_oracle_sample(w, x_cpu, w_idx_cpu, w_r_cpu, target_s, max_rows, threads=0):
    """Times the oracle on `rows` tokens: rotate + quantise each row, then its
    full output row of the quantised product, on `threads` threads (0: all).
    Returns (tokens/s, rows, seconds, threads used, oracle codes and s of the rows)."""
    import numpy as np

    import oracle

    perm, sign = oracle.plan(w.d, w.h, w.plan_seed)
    ca, ta = oracle.codebook(w.d, w.bits_a)
    cw, _ = oracle.codebook(w.d, w.bits_w)
    ca16 = oracle.round_bf16(ca)[1]
    cw16 = oracle.round_bf16(cw)[1]
    from rotation_bit_quantization_rpbh_b200 import binding as B

    iw = B.unpack_indices(w_idx_cpu, w.d, w.bits_w).numpy()
    r64 = w_r_cpu.float().numpy().astype(np.float64)
    oracle.set_num_threads(threads)
    used = oracle.num_threads()
    last = {}

    def run(rows):
        xs = x_cpu[:rows].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        q = oracle.quantize_rows(xs, w.h, perm, sign, ta, decision=32)
        last["y"] = oracle.qlinear(q["idx"], q["s"], iw, r64, ca16, cw16)
        dt = time.perf_counter() - t0
        last["q"] = q
        return dt

    try:
        rows = 2
        dt = run(rows)
        while dt < target_s * 0.5 and rows < max_rows:
            rows = min(max_rows, max(rows * 2, int(rows * target_s / max(dt, 1e-3))))
            dt = run(rows)
    finally:
        oracle.set_num_threads(0)
    return rows / dt, rows, dt, used, last


def cpu_baseline_block(w, x_cpu, w_idx_cpu, w_r_cpu, a_idx_gpu, s_gpu, y_gpu, target_s):
    """The oracle as the CPU baseline, on the host's cores: the layer on a
    bounded token sample (all threads, then one), the rotate-and-quantise
    pass over the full batch (all threads), and the parity of the GPU's
    codes, norms and product on the sampled rows."""
    import numpy as np

    import oracle
    from rotation_bit_quantization_rpbh_b200 import binding as B

    tok_s, rows, dt, thr, last = cpu_oracle_sample(w, x_cpu, w_idx_cpu, w_r_cpu, target_s, w.M)
    tok_1, rows_1, dt_1, _, _ = cpu_oracle_sample(w, x_cpu, w_idx_cpu, w_r_cpu, max(2.0, target_s / 4), w.M, 1)
    perm, sign = oracle.plan(w.d, w.h, w.plan_seed)
    _, ta = oracle.codebook(w.d, w.bits_a)
    x64 = x_cpu.float().numpy().astype(np.float64)
    t0 = time.perf_counter()
    oracle.quantize_rows(x64, w.h, perm, sign, ta, decision=32)
    t_full = time.perf_counter() - t0
    # parity on the sampled rows: codes, norms and product rows against the oracle
    gi = B.unpack_indices(a_idx_gpu[:rows].cpu(), w.d, w.bits_a).numpy()
    q = last["q"]
    mism = int((gi != q["idx"]).sum())
    s_rel = float(np.max(np.abs(s_gpu[:rows].cpu().numpy().astype(np.float64) - q["s"]) / np.maximum(q["s"], 1e-300)))
    yg = y_gpu[:rows].float().cpu().numpy().astype(np.float64)
    ref = last["y"]
    rel = float(np.linalg.norm(yg - ref) / max(np.linalg.norm(ref), 1e-300))
    return {"value": tok_s, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": f"{rows} tokens of {w.name}: rotate+quantise each row, then its full {w.N}-wide output row "
                      f"({dt:.1f} s on {thr} threads)",
            "single_core": {"value": tok_1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{rows_1} tokens, same work ({dt_1:.1f} s)"},
            "rpbh_quant_full_batch": {"seconds": t_full, "rows": w.M, "cores": thr,
                                      "gbs": rpbh_bytes(w) / t_full / 1e9,
                                      "note": "the oracle's rotate+split+quantise over all M rows (fp64, O(h) "
                                              "direct sums per output)"},
            "parity_on_sample": {"rows": rows, "code_mismatches": mism, "coordinates": rows * w.d,
                                 "s_max_rel_diff": s_rel, "product_rel_frobenius": rel,
                                 "note": "GPU codes (codes-mode launch) and GPU product rows against the oracle's "
                                         "own codes and fp64 product; mismatches are threshold ties within "
                                         "1e-6 relative (the parity tests check the band)"}}


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on bounded samples."""
    from rotation_bit_quantization_rpbh_b200 import inputs as I

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle

    w = I.WORKLOADS[args.workload]
    perm, sign = oracle.plan(w.d, w.h, w.plan_seed)
    ca, ta = oracle.codebook(w.d, w.bits_a)
    cw, tw = oracle.codebook(w.d, w.bits_w)
    ca16, cw16 = oracle.round_bf16(ca)[1], oracle.round_bf16(cw)[1]
    # offline weight pass (untimed): the oracle's own quantisation of W
    t_w = time.perf_counter()
    Wq = oracle.quantize_rows(I.make_w(w).float().numpy().astype(np.float64), w.h, perm, sign, tw, decision=32)
    t_w = time.perf_counter() - t_w
    threads = oracle.num_threads()
    # four rows per thread keep every thread of the oracle's row loop busy
    rows_per_step = max(1, min(w.M, 4 * threads))
    x = I.make_x(w, rows=np.arange(rows_per_step)).float().numpy().astype(np.float64)

    def step():
        q = oracle.quantize_rows(x, w.h, perm, sign, ta, decision=32)
        return oracle.qlinear(q["idx"], q["s"], Wq["idx"], Wq["s"], ca16, cw16)

    t = time.perf_counter()
    step()
    one = time.perf_counter() - t
    budget = 150.0
    while rows_per_step > threads and one * (args.steps + args.warmup) > budget:
        rows_per_step = max(threads, rows_per_step // 2)
        x = x[:rows_per_step]
        t = time.perf_counter()
        step()
        one = time.perf_counter() - t
    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t) / args.steps
    tok_s = rows_per_step / dt
    out = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "tokens_per_step": rows_per_step, "M": w.M, "d": w.d, "N": w.N, "h": w.h,
                      "bits_w": w.bits_w, "bits_a": w.bits_a, "parallelism": "replicas"},
           "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                            "sample": f"{rows_per_step} tokens per step of {w.name} ({rows_per_step // threads} per "
                                      f"thread; rotate+quantise the rows, then their full {w.N}-wide output rows); "
                                      f"offline weight pass {t_w:.1f} s untimed"},
           "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


class Layer:
    """One workload's layer on the device: inputs, the offline weight pass,
    the workspace and the two timed calls of a step (quantiser, product) in
    the chosen schedule, plus a codes-mode quantiser launch."""

    def __init__(self, w, dev, schedule, fp8):
        import torch

        from rotation_bit_quantization_rpbh_b200 import binding as B
        from rotation_bit_quantization_rpbh_b200 import inputs as I

        self.w, self.schedule, self.fp8 = w, schedule, fp8
        self.x_cpu = I.make_x(w)
        W_cpu = I.make_w(w)
        self.plan = B.rpbh_plan(w.d, w.h, w.plan_seed)
        self.cb_a, self.cb_w = B.codebook(w.d, w.bits_a), B.codebook(w.d, w.bits_w)
        self.x = self.x_cpu.to(dev)
        self.w_idx, self.w_r = B.quantize_weights(self.plan, self.cb_w, W_cpu.to(dev))  # offline pass, untimed
        del W_cpu
        self.ws = torch.empty(max(B.qlinear_workspace(w.M, w.d, w.bits_a), B.qlinear_workspace_values(w.M, w.d)),
                              dtype=torch.uint8, device=dev)
        ws = self.ws
        if schedule == "values":
            vb = 1 if fp8 else 2
            self.a_in = ws[: w.M * w.d * vb].view(w.M, w.d * vb)
            if not fp8:
                self.a_in = self.a_in.view(torch.bfloat16)
            s_off = (w.M * w.d * vb + 255) // 256 * 256
        else:
            packed = B.packed_row_bytes(w.d, w.bits_a)
            self.a_in = ws[: w.M * packed].view(w.M, packed)
            s_off = (w.M * packed + 255) // 256 * 256
        self.s = ws[s_off: s_off + 4 * w.M].view(torch.float32)
        self.y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
        self.codes = torch.empty((w.M, B.packed_row_bytes(w.d, w.bits_a)), dtype=torch.uint8, device=dev)
        self.s_codes = torch.empty(w.M, dtype=torch.float32, device=dev)

    def quant(self, stream):
        from rotation_bit_quantization_rpbh_b200 import binding as B

        if self.schedule == "values":
            B.quantize_acts_values(self.plan, self.cb_a, self.x, self.a_in, self.s, stream=stream, fp8=self.fp8)
        else:
            B.quantize_acts(self.plan, self.cb_a, self.x, self.a_in, self.s, stream=stream)

    def gemm(self, stream):
        from rotation_bit_quantization_rpbh_b200 import binding as B

        if self.schedule == "values":
            B.qgemm_values(self.cb_w, self.a_in, self.s, self.w_idx, self.w_r, y=self.y, stream=stream, fp8=self.fp8)
        else:
            (B.qgemm_fp8 if self.fp8 else B.qgemm)(self.cb_a, self.cb_w, self.a_in, self.s, self.w_idx, self.w_r,
                                                    y=self.y, stream=stream)

    def quant_codes(self, stream):
        from rotation_bit_quantization_rpbh_b200 import binding as B

        B.quantize_acts(self.plan, self.cb_a, self.x, self.codes, self.s_codes, stream=stream)


def time_layer(L, steps, warmup, flush, stream):
    """Event times (ms) of the whole step (quantiser then product, with
    nothing between them in the stream, so the product's programmatic launch
    overlaps the quantiser's end), then of the quantiser alone and of the
    product alone, each over `steps` launches, L2 flushed before each
    outside the events.  Returns (quantiser, product, step) lists."""
    import torch

    for _ in range(max(3, warmup)):
        flush.zero_()
        L.quant(stream)
        L.gemm(stream)
    torch.cuda.synchronize()

    def timed(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) for e0, e1 in ev]

    t_step = timed(lambda: (L.quant(stream), L.gemm(stream)))
    t_rpbh = timed(lambda: L.quant(stream))
    t_gemm = timed(lambda: L.gemm(stream))
    return t_rpbh, t_gemm, t_step


def time_layer_graph(L, steps, flush, stream):
    """Event time (ms) per replay of the step captured in a CUDA graph (the
    two launches and their programmatic dependency), L2 flushed before each
    replay outside the events."""
    import numpy as np
    import torch

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap = torch.cuda.current_stream()
        L.quant(cap)
        L.gemm(cap)
    for _ in range(3):
        flush.zero_()
        graph.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    del graph
    return float(np.mean([e0.elapsed_time(e1) for e0, e1 in ev]))


def time_codes_quantiser(L, steps, flush, stream):
    """Event time (ms) per launch of the codes-mode quantiser (the method's
    packed output), L2 flushed before each launch."""
    import numpy as np
    import torch

    for _ in range(3):
        flush.zero_()
        L.quant_codes(stream)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        L.quant_codes(stream)
        e1.record(stream)
    torch.cuda.synchronize()
    return float(np.mean([e0.elapsed_time(e1) for e0, e1 in ev]))


def host_call_overhead(L, stream, calls):
    """Host time per oq_qlinear call (argument checks, marshalling and the
    two launches), measured over `calls` back-to-back calls without a sync."""
    import torch

    from rotation_bit_quantization_rpbh_b200 import binding as B

    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(calls):
        B.qlinear(L.plan, L.cb_a, L.cb_w, L.x, L.w_idx, L.w_r, y=L.y, workspace=L.ws, stream=stream, fp8=L.fp8)
    t1 = time.perf_counter()
    torch.cuda.synchronize()
    return (t1 - t0) / calls * 1e6


def rooflines(w, peaks, fp8, ms_gemm, ms_rpbh, ms_codes, schedule, kernel_names):
    flops = 2.0 * w.M * w.N * w.d
    mma_peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    gemm_tflops = flops / (ms_gemm * 1e-3) / 1e12
    rb = rpbh_bytes(w)
    gemm_key, rpbh_key = kernel_names
    out = {
        "roofline": {"bound": "tensor", "kernel": gemm_key, "achieved": gemm_tflops, "peak": mma_peak,
                     "unit": "TFLOP/s", "frac": gemm_tflops / mma_peak,
                     "traffic": committed_traffic(gemm_key, w.name),
                     "peak_source": peaks["source"] + (" bf16 (burst) x nominal fp8/bf16 ratio 2" if fp8 else
                                                       " (burst)"),
                     "algorithmic": f"2*M*N*d = {flops:.4g} flop per launch"},
        "roofline_rpbh": {"bound": "hbm", "kernel": rpbh_key, "achieved": rb / (ms_rpbh * 1e-3) / 1e9,
                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": rb / (ms_rpbh * 1e-3) / 1e9 / peaks["hbm_gbs"],
                          "traffic": committed_traffic(rpbh_key, w.name),
                          "algorithmic": f"M*(d*in_bytes + packed codes + 4) = {rb} B per launch (the method's "
                                         f"output; the {schedule} schedule's launch writes "
                                         f"{'centroid values' if schedule == 'values' else 'the codes'})"},
        "roofline_rpbh_codes": {"bound": "hbm", "kernel": "rpbh_quant", "achieved": rb / (ms_codes * 1e-3) / 1e9,
                                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": rb / (ms_codes * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "traffic": committed_traffic("rpbh_quant", w.name),
                                "algorithmic": f"{rb} B per launch", "ms": ms_codes,
                                "note": "the quantiser writing the packed codes (oq_quantize_acts), timed alone"},
    }
    return out, gemm_tflops


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from rotation_bit_quantization_rpbh_b200 import binding as B
    from rotation_bit_quantization_rpbh_b200 import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CPU oracle is the reference arm: --impl reference)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    B.lib()

    w = I.WORKLOADS[args.workload]
    schedule = "values" if args.schedule == "auto" else args.schedule  # the one oq_qlinear takes
    L = Layer(w, dev, schedule, args.fp8)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2 (126 MB)
    stream = torch.cuda.current_stream()

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        L.quant(stream)
        L.gemm(stream)
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("start")
    t_rpbh, t_gemm, t_step = time_layer(L, args.steps, 0, flush, stream)  # step first, then each kernel alone
    if world > 1:
        dist.barrier()
    sampler.mark("stop")
    clocks = sampler.stop()
    if B.device_status() != 0:
        raise SystemExit("a kernel reported a timeout")
    ms, ms_rpbh, ms_gemm = reduce_max([float(np.mean(t_step)), float(np.mean(t_rpbh)), float(np.mean(t_gemm))],
                                      world, dev)
    ms_codes = reduce_max([time_codes_quantiser(L, max(5, min(args.steps, 20)), flush, stream)], world, dev)[0]
    ms_graph = reduce_max([time_layer_graph(L, max(5, min(args.steps, 20)), flush, stream)], world, dev)[0]

    # end to end through the public one-call API with host buffers: every
    # step copies its x in from pinned host memory, runs oq_qlinear and
    # copies y out, pipelined two deep on three streams (copy-in of step
    # i+1 and copy-out of step i-1 overlap the layer of step i)
    e2e = None
    if not args.no_e2e:
        x_pin = L.x_cpu.pin_memory()
        nbuf = 2
        xs = [torch.empty_like(L.x) for _ in range(nbuf)]
        ys = [torch.empty_like(L.y) for _ in range(nbuf)]
        # oq_qlinear takes its preferred schedule when the workspace holds it;
        # a codes-sized workspace makes it take the codes schedule
        ws_e2e = L.ws.numel() if schedule == "values" else B.qlinear_workspace(w.M, w.d, w.bits_a)
        wss = [torch.empty(ws_e2e, dtype=torch.uint8, device=dev) for _ in range(nbuf)]
        y_pins = [torch.empty((w.M, w.N), dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(nbuf)]
        ev_cmp = [torch.cuda.Event() for _ in range(nbuf)]
        ev_out = [torch.cuda.Event() for _ in range(nbuf)]
        for b in range(nbuf):  # nothing pending on any buffer yet
            ev_cmp[b].record(s_cmp)
            ev_out[b].record(s_out)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_warm = max(3, args.warmup)
        for it in range(n_warm + args.steps):
            if it == n_warm:
                torch.cuda.synchronize()
                if world > 1:
                    dist.barrier()
                e0.record(s_in)
            b = it % nbuf
            s_in.wait_event(ev_cmp[b])  # the layer that last read xs[b] is done
            with torch.cuda.stream(s_in):
                xs[b].copy_(x_pin, non_blocking=True)
            ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])  # the copy-out that last read ys[b] is done
            B.qlinear(L.plan, L.cb_a, L.cb_w, xs[b], L.w_idx, L.w_r, y=ys[b], workspace=wss[b], stream=s_cmp,
                      fp8=args.fp8)
            ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                y_pins[b].copy_(ys[b], non_blocking=True)
            ev_out[b].record(s_out)
        s_out.wait_stream(s_in)
        s_out.wait_stream(s_cmp)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = reduce_max([e0.elapsed_time(e1) / args.steps], world, dev)[0]
        e2e = {"value": job_throughput(world, w.M, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(L.x_cpu.numel() * L.x_cpu.element_size()),
               "d2h_bytes_per_step": int(L.y.numel() * L.y.element_size()), "ms_per_step": e2e_ms,
               "pipeline": "copy-in, oq_qlinear and copy-out on three streams, two buffers deep",
               "schedule": schedule}

    peaks = measured_peaks()
    gemm_key = ("qgemm_values" if schedule == "values" else "qgemm") + ("_fp8" if args.fp8 else "")
    rpbh_key = "rpbh_quant" + (("_values_fp8" if args.fp8 else "_values") if schedule == "values" else "")
    roof, gemm_tflops = rooflines(w, peaks, args.fp8, ms_gemm, ms_rpbh, ms_codes, schedule, (gemm_key, rpbh_key))
    if world == 1:
        # context for the per-launch figure: the launch floor every event time
        # contains, and the quantiser's rate over 2x-8x the workload's rows
        # (the slope: the cost per row once the fixed cost is amortised)
        k_sw = max(5, min(args.steps, 10))
        srows, per_row, _ = quant_sweep_rows(w, L.plan, L.cb_a, L.x, [2 * w.M, 4 * w.M, 8 * w.M], flush, stream,
                                             k_sw, 3, values=False)
        roof["roofline_rpbh_codes"]["launch_floor_us"] = launch_floor_us(flush, stream, k_sw)
        roof["roofline_rpbh_codes"]["steady_state"] = steady_fit(srows, per_row, peaks["hbm_gbs"], 2 * w.M)
    flops = 2.0 * w.M * w.N * w.d
    out = {
        "metric": METRIC, "value": job_throughput(world, w.M, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "d": w.d, "N": w.N, "h": w.h, "bits_w": w.bits_w,
                   "bits_a": w.bits_a, "x_dtype": w.x_dtype, "tokens_per_gpu": w.M, "global_batch": world * w.M,
                   "parallelism": f"dp{world} (replicated packed W, no collective)", "schedule": schedule,
                   "l2": "flushed (256 MB write) before every timed step, outside the events"},
        "tflops": flops / (ms * 1e-3) / 1e12,
        "breakdown": {"rpbh_quant_ms": ms_rpbh, "qgemm_ms": ms_gemm, "qgemm_tflops": gemm_tflops,
                      "rpbh_quant_gbs": roof["roofline_rpbh"]["achieved"], "rpbh_quant_codes_ms": ms_codes,
                      "overlap_ms": ms_rpbh + ms_gemm - ms, "graph_step_ms": ms_graph,
                      "note": "the step is timed as one unit (the product launches programmatically and overlaps "
                              "the quantiser's end); each kernel is then timed alone over the same number of "
                              "launches, L2 flushed before each; graph_step_ms: the same step captured in a CUDA "
                              "graph and replayed"},
        **roof,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "e2e": e2e,
    }
    # host time per oq_qlinear call: flat in the number of calls (no per-call
    # device allocation, synchronisation or tensor-map encoding)
    out["host_us_per_call"] = {str(n): host_call_overhead(L, stream, n) for n in (10, 100)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        L.quant_codes(stream)
        torch.cuda.synchronize()
        out["cpu_baseline"] = cpu_baseline_block(w, L.x_cpu, L.w_idx.cpu(), L.w_r.cpu(), L.codes, L.s_codes, L.y,
                                                 args.cpu_seconds)
    # the other large workloads, each timed the same way on this GPU
    if world == 1 and not args.no_per_workload:
        per = {}
        for name in I.ORDER:
            w2 = I.WORKLOADS[name]
            if name == w.name or w2.M < 1024:
                continue
            L2 = Layer(w2, dev, schedule, args.fp8)
            k2 = max(5, min(args.steps, 20))
            tr, tg, ts = time_layer(L2, k2, 3, flush, stream)
            mc = time_codes_quantiser(L2, k2, flush, stream)
            if B.device_status() != 0:
                raise SystemExit("a kernel reported a timeout")
            r2, gt2 = rooflines(w2, peaks, args.fp8, float(np.mean(tg)), float(np.mean(tr)), mc, schedule,
                                (gemm_key, rpbh_key))
            per[name] = {"tokens_per_s": w2.M / (float(np.mean(ts)) * 1e-3), "ms_per_step": float(np.mean(ts)),
                         "steps": k2, "qgemm_tflops": gt2, "qgemm_frac": r2["roofline"]["frac"],
                         "rpbh_quant_ms": float(np.mean(tr)), "rpbh_quant_gbs": r2["roofline_rpbh"]["achieved"],
                         "rpbh_quant_frac": r2["roofline_rpbh"]["frac"], "rpbh_quant_codes_ms": mc,
                         "rpbh_quant_codes_frac": r2["roofline_rpbh_codes"]["frac"]}
            del L2
            torch.cuda.empty_cache()
        out["per_workload"] = per
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def full_rht_block(d):
    """Full RHT: one Walsh-Hadamard block over all of d.  Sylvester matrices
    exist for powers of two only, so for other d the largest power-of-two
    block that divides d (3072 -> 1024, 12288 -> 4096, 1536 -> 512)."""
    h = 1
    while d % (2 * h) == 0 and 2 * h <= 16384:
        h *= 2
    return h


def run_ablation(args):
    """The page's rotation ablation on one GPU: the fused rotate+quantise
    kernel and the rotation alone (oq_rpbh_apply) with the RPBH plan, the
    Block-RHT plan (no permutation: each block read contiguously), the Full
    RHT plan (no permutation, one block over d, or the largest power-of-two
    block of d), and a dense Haar rotation (a cuBLAS bf16 GEMM against a
    random orthogonal d x d matrix).  Median device time per call over
    --steps calls, L2 flushed before each."""
    import numpy as np
    import torch

    from rotation_bit_quantization_rpbh_b200 import binding as B
    from rotation_bit_quantization_rpbh_b200 import inputs as I

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --ablation needs a CUDA device")
    dev = torch.device("cuda", 0)
    w = I.WORKLOADS[args.workload]
    x = I.make_x(w).to(dev)
    cb_a = B.codebook(w.d, w.bits_a)
    hf = full_rht_block(w.d)
    plans = {"rpbh": B.rpbh_plan(w.d, w.h, w.plan_seed),
             "block_rht": B.rotation_plan(w.d, w.h, w.plan_seed, B.OQ_ROT_BLOCK_RHT),
             "full_rht": B.rotation_plan(w.d, hf, w.plan_seed, B.OQ_ROT_BLOCK_RHT)}
    a_idx = torch.empty((w.M, B.packed_row_bytes(w.d, w.bits_a)), dtype=torch.uint8, device=dev)
    s = torch.empty(w.M, dtype=torch.float32, device=dev)
    x_rot = torch.empty((w.M, w.d), dtype=torch.float32, device=dev)
    # Haar-distributed orthogonal matrix: QR of a Gaussian matrix with the
    # signs of R's diagonal folded into Q (Mezzadri 2007)
    g = torch.Generator(device=dev).manual_seed(w.plan_seed)
    q, r = torch.linalg.qr(torch.randn(w.d, w.d, generator=g, device=dev, dtype=torch.float32))
    q = q * torch.sign(torch.diagonal(r)).unsqueeze(0)
    haar_t = q.t().contiguous().to(torch.bfloat16)
    xb = x.to(torch.bfloat16)
    y_haar = torch.empty((w.M, w.d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    calls = {}
    for name, pl in plans.items():
        calls[f"{name}_quant"] = (lambda pl=pl: B.quantize_acts(pl, cb_a, x, a_idx, s, stream=stream))
        calls[f"{name}_rotate"] = (lambda pl=pl: B.rpbh_apply(pl, x, x_rot, s, stream=stream))
    calls["haar_rotate_cublas"] = lambda: torch.matmul(xb, haar_t, out=y_haar)

    # the same two plans through one kernel family each: the team kernel
    # (the Block-RHT plan's contiguous reads against the RPBH gather) and
    # the warp-group kernel (both plans gathered through their tables)
    def forced(family, fn):
        def call():
            B.debug_rpbh_kernel(family)
            try:
                fn()
            finally:
                B.debug_rpbh_kernel(0)
        return call

    calls["rpbh_quant_teams"] = forced(B.RPBH_KERNEL_TEAMS, calls["rpbh_quant"])
    calls["rpbh_quant_groups"] = forced(B.RPBH_KERNEL_GROUPS, calls["rpbh_quant"])
    calls["block_rht_quant_groups"] = forced(B.RPBH_KERNEL_GROUPS, calls["block_rht_quant"])
    ms = {}
    for name, fn in calls.items():
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        ms[name] = float(np.median([e0.elapsed_time(e1) for e0, e1 in ev]))
    if B.device_status() != 0:
        raise SystemExit("a kernel reported a timeout")
    out = {
        "metric": "rotation ablation: device ms per call (median)",
        "workload": w.name, "M": w.M, "d": w.d, "h": w.h, "full_rht_h": hf, "bits_a": w.bits_a, "steps": args.steps,
        "ms": ms,
        "ratios": {
            "rpbh_over_block_rht_quant": ms["rpbh_quant"] / ms["block_rht_quant"],
            "rpbh_over_block_rht_quant_team_kernel": ms["rpbh_quant_teams"] / ms["block_rht_quant"],
            "rpbh_over_block_rht_quant_group_kernel": ms["rpbh_quant_groups"] / ms["block_rht_quant_groups"],
            "rpbh_over_block_rht_rotate": ms["rpbh_rotate"] / ms["block_rht_rotate"],
            "full_rht_over_rpbh_rotate": ms["full_rht_rotate"] / ms["rpbh_rotate"],
            "haar_over_rpbh_rotate": ms["haar_rotate_cublas"] / ms["rpbh_rotate"],
            "haar_over_block_rht_rotate": ms["haar_rotate_cublas"] / ms["block_rht_rotate"],
            "haar_over_full_rht_rotate": ms["haar_rotate_cublas"] / ms["full_rht_rotate"],
            # the layer's cost of a dense rotation: the Haar GEMM, then a quantise
            # pass over its output (the Block-RHT plan's launch stands in for a
            # quantiser without a transform), against the fused RPBH launch
            "haar_plus_quant_over_rpbh_quant": (ms["haar_rotate_cublas"] + ms["block_rht_quant"]) / ms["rpbh_quant"],
        },
        "note": "rotate = oq_rpbh_apply (fp32 x' and norms out); quant = the fused rotate+split+quantise kernel "
                "(packed codes out), each plan on its default kernel; _teams / _groups = forced onto the team or "
                "the warp-group kernel; Block-RHT and Full RHT read each block contiguously (no permutation) "
                "except on the warp-group kernel, which gathers through the identity table; "
                "haar = bf16 x @ Q^T with a Haar-random Q, bf16 out (cuBLAS); L2 flushed before every call",
    }
    print(json.dumps(out), flush=True)


def _median_event_us(fn, flush, stream, steps, warmup):
    """Median event time (us) of fn() over `steps` calls, L2 flushed (256 MB
    write, outside the events) before each."""
    import numpy as np
    import torch

    for _ in range(max(3, warmup)):
        flush.zero_()
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return float(np.median([e0.elapsed_time(e1) for e0, e1 in ev])) * 1e3


def launch_floor_us(flush, stream, steps):
    """A one-element torch kernel timed like the kernels: the fixed launch
    and event cost that every per-launch time here contains."""
    import torch

    one = torch.zeros(1, device=flush.device)
    return _median_event_us(lambda: one.add_(1.0), flush, stream, steps, 3)


def quant_sweep_rows(w, plan, cb, x0, Ms, flush, stream, steps, warmup, values=True):
    """Quantiser event times at M rows each (the workload's rows repeated)."""
    import torch

    from rotation_bit_quantization_rpbh_b200 import binding as B

    per_row = w.d * x0.element_size() + B.packed_row_bytes(w.d, w.bits_a) + 4  # §8(d) bytes per token
    peak = measured_peaks()["hbm_gbs"]
    rows = []
    for M in Ms:
        reps = (M + x0.shape[0] - 1) // x0.shape[0]
        x = x0.repeat(reps, 1)[:M].contiguous()
        idx = torch.empty((M, B.packed_row_bytes(w.d, w.bits_a)), dtype=torch.uint8, device=x0.device)
        s = torch.empty(M, dtype=torch.float32, device=x0.device)
        tc = _median_event_us(lambda: B.quantize_acts(plan, cb, x, idx, s, stream=stream), flush, stream, steps, warmup)
        r = {"M": M, "codes_us": tc, "codes_gbs": M * per_row / (tc * 1e-6) / 1e9}
        r["codes_frac"] = r["codes_gbs"] / peak
        if values:
            val = torch.empty((M, w.d), dtype=torch.bfloat16, device=x0.device)
            r["values_us"] = _median_event_us(lambda: B.quantize_acts_values(plan, cb, x, val, s, stream=stream),
                                              flush, stream, steps, warmup)
            del val
        rows.append(r)
        del x, idx, s
    return rows, per_row, peak


def steady_fit(rows, per_row, peak, m_min):
    """Least-squares line through codes_us against M for M >= m_min: the
    per-row cost as a rate (GB/s and fraction of the peak) and the fixed
    cost (intercept)."""
    import numpy as np

    big = [r for r in rows if r["M"] >= m_min]
    if len(big) < 2:
        return None
    k, c0 = np.polyfit(np.array([r["M"] for r in big], dtype=np.float64),
                       np.array([r["codes_us"] for r in big], dtype=np.float64), 1)
    gbs = per_row / (k * 1e-6) / 1e9
    return {"us_per_row": float(k), "intercept_us": float(c0), "steady_gbs": gbs, "steady_frac": gbs / peak,
            "fit_M": [r["M"] for r in big]}


def run_quant_sweep(args):
    """The quantiser alone (codes and bf16 values modes) at the workload's d,
    h and bits over a range of M: the workload's own rows repeated.  Event
    time per launch (median of --steps, L2 flushed before each), beside a
    one-element torch kernel timed the same way (the launch floor of this
    measurement).  The slope over the largest M gives the steady-state
    rate, free of the fixed launch and ramp cost."""
    import torch

    from rotation_bit_quantization_rpbh_b200 import binding as B
    from rotation_bit_quantization_rpbh_b200 import inputs as I

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --quant-sweep needs a CUDA device")
    dev = torch.device("cuda", 0)
    w = I.WORKLOADS[args.workload]
    x0 = I.make_x(w).to(dev)
    plan = B.rpbh_plan(w.d, w.h, w.plan_seed)
    cb = B.codebook(w.d, w.bits_a)
    cb.upload()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    floor = launch_floor_us(flush, stream, args.steps)
    Ms = sorted(M for M in {148, 592, 2048, w.M, 2 * w.M, 4 * w.M, 8 * w.M} if M * w.d * 2 * 3 <= (3 << 30))
    rows, per_row, peak = quant_sweep_rows(w, plan, cb, x0, Ms, flush, stream, args.steps, args.warmup)
    if B.device_status() != 0:
        raise SystemExit("a kernel reported a timeout")
    print(json.dumps({"metric": "quantiser event time against M", "workload": w.name, "d": w.d, "h": w.h,
                      "bits_a": w.bits_a, "steps": args.steps, "launch_floor_us": floor,
                      "bytes_per_row": per_row, "peak_gbs": peak, "rows": rows,
                      "fit_codes": steady_fit(rows, per_row, peak, 2 * w.M),
                      "note": "event time per launch, L2 flushed (256 MB write) before each; launch_floor_us is a "
                              "one-element torch kernel timed the same way; fit over M >= 2x the workload's M"}))


def run_gemm_sweep(args):
    """The A-values product alone (bf16, or e4m3 with --fp8) at the
    workload's d, N and bits over a range of M: the workload's rows
    repeated, quantised once.  Event time per launch (median of --steps, L2
    flushed before each).  A pair of SMs takes one 256 x 256 tile at a time,
    so the time grows in rounds of (SMs / 2) tiles; the slope over the
    largest M gives the steady per-round rate, free of the launch floor, the
    pipeline fill and drain and the partial last round."""
    import numpy as np
    import torch

    from rotation_bit_quantization_rpbh_b200 import binding as B
    from rotation_bit_quantization_rpbh_b200 import inputs as I

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --gemm-sweep needs a CUDA device")
    dev = torch.device("cuda", 0)
    w = I.WORKLOADS[args.workload]
    x0 = I.make_x(w).to(dev)
    plan = B.rpbh_plan(w.d, w.h, w.plan_seed)
    cb_a, cb_w = B.codebook(w.d, w.bits_a), B.codebook(w.d, w.bits_w)
    w_idx, w_r = B.quantize_weights(plan, cb_w, I.make_w(w).to(dev))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    pairs = torch.cuda.get_device_properties(dev).multi_processor_count // 2
    peak = measured_peaks()["bf16_tflops"] * (2 if args.fp8 else 1)
    rows = []
    for M in sorted({w.M // 4, w.M // 2, w.M, 2 * w.M, 4 * w.M, 8 * w.M}):
        if M < 256 or M * (w.d * 2 + w.N * 2) > (3 << 30):
            continue
        x = x0.repeat((M + w.M - 1) // w.M, 1)[:M].contiguous()
        val, s = B.quantize_acts_values(plan, cb_a, x, fp8=args.fp8)
        y = torch.empty((M, w.N), dtype=torch.bfloat16, device=dev)
        us = _median_event_us(lambda: B.qgemm_values(cb_w, val, s, w_idx, w_r, y=y, stream=stream, fp8=args.fp8),
                              flush, stream, args.steps, args.warmup)
        tiles = ((M + 255) // 256) * ((w.N + 255) // 256)
        tf = 2.0 * M * w.N * w.d / (us * 1e-6) / 1e12
        rows.append({"M": M, "us": us, "tiles": tiles, "rounds": tiles / pairs, "tflops": tf, "frac": tf / peak})
        del x, val, s, y
    if B.device_status() != 0:
        raise SystemExit("a kernel reported a timeout")
    fit = None
    big = [r for r in rows if r["M"] >= 2 * w.M]
    if len(big) >= 2:
        k, c0 = np.polyfit(np.array([r["rounds"] for r in big]), np.array([r["us"] for r in big]), 1)
        flop_round = 2.0 * pairs * 256 * 256 * w.d
        fit = {"us_per_round": float(k), "intercept_us": float(c0), "steady_tflops": flop_round / (k * 1e-6) / 1e12,
               "steady_frac": flop_round / (k * 1e-6) / 1e12 / peak, "fit_M": [r["M"] for r in big]}
    print(json.dumps({"metric": "A-values product event time against M", "workload": w.name, "d": w.d, "N": w.N,
                      "bits_w": w.bits_w, "fp8": args.fp8, "sm_pairs": pairs, "steps": args.steps,
                      "peak_tflops": peak, "rows": rows, "fit": fit,
                      "note": "event time per launch, L2 flushed (256 MB write) before each; a round is one "
                              "256 x 256 tile per SM pair; fit over M >= 2x the workload's M"}))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.ablation:
        run_ablation(args)
    elif args.quant_sweep:
        run_quant_sweep(args)
    elif args.gemm_sweep:
        run_gemm_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
