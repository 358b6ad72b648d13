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
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline sample")
    ap.add_argument("--fp8", action="store_true",
                    help="time the fp8 variant of the product (oq_qgemm_fp8: e4m3 centroid values)")
    ap.add_argument("--schedule", default="auto", choices=["auto", "codes", "values"],
                    help="layer schedule timed: activation codes decoded in the GEMM, or centroid values written by "
                         "the quantiser and streamed into the GEMM; auto = the one oq_qlinear takes")
    ap.add_argument("--ablation", action="store_true",
                    help="time the rotation ablation (RPBH, Block-RHT, dense Haar) on --workload instead of the layer")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


KERNEL_SOURCES = {"qgemm": "qgemm.cu", "qgemm_fp8": "qgemm.cu", "qgemm_values": "qgemm.cu",
                  "qgemm_values_fp8": "qgemm.cu", "rpbh_quant": "rpbh_quant.cu", "rpbh_quant_values": "rpbh_quant.cu",
                  "rpbh_quant_values_fp8": "rpbh_quant.cu"}


def committed_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if one exists for
    this kernel and workload and the kernel source is unchanged since the
    counters were taken (null otherwise)."""
    import hashlib

    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f).get(kernel, {})
    src = os.path.join(ROOT, "rotation_bit_quantization_rpbh_b200", "csrc", KERNEL_SOURCES[kernel])
    with open(src, encoding="utf-8") as f:
        if hashlib.md5(code_only(f.read()).encode()).hexdigest() != j.get("code_md5"):
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


def rpbh_bytes(w, schedule="codes", fp8=False):
    """Algorithmic bytes of one quantiser launch: x read, then the packed
    codes (codes schedule) or the centroid values (values schedule: 2 bytes
    each, 1 in e4m3) written, plus s."""
    esize = 4 if w.x_dtype == "f32" else 2
    if schedule == "values":
        out = w.d * (1 if fp8 else 2)
    else:
        out = w.d if w.bits_a == 6 else w.d * w.bits_a // 8
    return w.M * (w.d * esize + out + 4)


def cpu_oracle_sample(w, x_cpu, w_idx_cpu, w_r_cpu, target_s, max_rows):
    """Times the oracle on `rows` tokens: rotate + quantise each row, then its
    full output row of the quantised product.  Returns (tokens/s, rows, s, threads)."""
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

    def run(rows):
        xs = x_cpu[:rows].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        q = oracle.quantize_rows(xs, w.h, perm, sign, ta, decision=32)
        oracle.qlinear(q["idx"], q["s"], iw, r64, ca16, cw16)
        return time.perf_counter() - t0

    rows = 2
    dt = run(rows)
    while dt < target_s * 0.5 and rows < max_rows:
        rows = min(max_rows, max(rows * 2, int(rows * target_s / max(dt, 1e-3))))
        dt = run(rows)
    return rows / dt, rows, dt, oracle.num_threads()


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on bounded samples."""
    from rotation_bit_quantization_rpbh_b200 import inputs as I

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle
    from rotation_bit_quantization_rpbh_b200 import binding as B

    w = I.WORKLOADS[args.workload]
    perm, sign = oracle.plan(w.d, w.h, w.plan_seed)
    ca, ta = oracle.codebook(w.d, w.bits_a)
    cw, tw = oracle.codebook(w.d, w.bits_w)
    ca16, cw16 = oracle.round_bf16(ca)[1], oracle.round_bf16(cw)[1]
    # offline weight pass (untimed): the oracle's own quantisation of W
    t_w = time.perf_counter()
    Wq = oracle.quantize_rows(I.make_w(w).float().numpy().astype(np.float64), w.h, perm, sign, tw, decision=32)
    t_w = time.perf_counter() - t_w
    rows_per_step = max(1, min(w.M, 8))
    x = I.make_x(w, rows=np.arange(rows_per_step)).float().numpy().astype(np.float64)

    def step():
        q = oracle.quantize_rows(x, w.h, perm, sign, ta, decision=32)
        return oracle.qlinear(q["idx"], q["s"], Wq["idx"], Wq["s"], ca16, cw16)

    t = time.perf_counter()
    step()
    one = time.perf_counter() - t
    budget = 150.0
    while rows_per_step > 1 and one * (args.steps + args.warmup) > budget:
        rows_per_step //= 2
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
           "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                            "sample": f"{rows_per_step} tokens per step of {w.name} (rotate+quantise the rows, "
                                      f"then their full {w.N}-wide output rows); offline weight pass "
                                      f"{t_w:.1f} s untimed"},
           "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


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
    x_cpu = I.make_x(w)
    W_cpu = I.make_w(w)
    plan = B.rpbh_plan(w.d, w.h, w.plan_seed)
    cb_a, cb_w = B.codebook(w.d, w.bits_a), B.codebook(w.d, w.bits_w)
    x = x_cpu.to(dev)
    w_idx, w_r = B.quantize_weights(plan, cb_w, W_cpu.to(dev))  # offline pass, untimed
    schedule = "values" if args.schedule == "auto" else args.schedule  # the one oq_qlinear takes
    ws = torch.empty(max(B.qlinear_workspace(w.M, w.d, w.bits_a), B.qlinear_workspace_values(w.M, w.d)),
                     dtype=torch.uint8, device=dev)
    if schedule == "values":
        vb = 1 if args.fp8 else 2
        a_in = ws[: w.M * w.d * vb].view(w.M, w.d * vb)
        if not args.fp8:
            a_in = a_in.view(torch.bfloat16)
        s_off = (w.M * w.d * vb + 255) // 256 * 256
    else:
        packed = w.d if w.bits_a == 6 else w.d * w.bits_a // 8
        a_in = ws[: w.M * packed].view(w.M, packed)
        s_off = (w.M * packed + 255) // 256 * 256
    s = ws[s_off: s_off + 4 * w.M].view(torch.float32)
    y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2 (126 MB)
    stream = torch.cuda.current_stream()

    if schedule == "values":
        def quant():
            B.quantize_acts_values(plan, cb_a, x, a_in, s, stream=stream, fp8=args.fp8)

        def gemm():
            B.qgemm_values(cb_w, a_in, s, w_idx, w_r, y=y, stream=stream, fp8=args.fp8)
    else:
        def quant():
            B.quantize_acts(plan, cb_a, x, a_in, s, stream=stream)

        def gemm():
            (B.qgemm_fp8 if args.fp8 else B.qgemm)(cb_a, cb_w, a_in, s, w_idx, w_r, y=y, stream=stream)

    def step():
        quant()
        gemm()

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("start")
    for i in range(args.steps):
        flush.zero_()  # cold L2 for every step (outside the events)
        ev[i][0].record(stream)
        quant()
        ev[i][1].record(stream)
        gemm()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler.mark("stop")
    clocks = sampler.stop()
    if B.device_status() != 0:
        raise SystemExit("a kernel reported a timeout")

    t_rpbh = [e[0].elapsed_time(e[1]) for e in ev]
    t_gemm = [e[1].elapsed_time(e[2]) for e in ev]
    t_step = [e[0].elapsed_time(e[2]) for e in ev]
    ms = float(np.mean(t_step))
    ms_rpbh = float(np.mean(t_rpbh))
    ms_gemm = float(np.mean(t_gemm))
    ms, ms_rpbh, ms_gemm = reduce_max([ms, ms_rpbh, ms_gemm], world, dev)

    # end to end through the public one-call API with host buffers: every
    # step copies its x in from pinned host memory, runs oq_qlinear and
    # copies y out, pipelined two deep on three streams (copy-in of step
    # i+1 and copy-out of step i-1 overlap the layer of step i)
    e2e = None
    if not args.no_e2e:
        x_pin = x_cpu.pin_memory()
        nbuf = 2
        xs = [torch.empty_like(x) for _ in range(nbuf)]
        ys = [torch.empty_like(y) for _ in range(nbuf)]
        # oq_qlinear takes its preferred schedule when the workspace holds it;
        # a codes-sized workspace makes it take the codes schedule
        e2e_schedule = schedule
        ws_e2e = ws.numel() if e2e_schedule == "values" else B.qlinear_workspace(w.M, w.d, w.bits_a)
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
            B.qlinear(plan, cb_a, cb_w, xs[b], w_idx, w_r, y=ys[b], workspace=wss[b], stream=s_cmp, fp8=args.fp8)
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
               "h2d_bytes_per_step": int(x_cpu.numel() * x_cpu.element_size()),
               "d2h_bytes_per_step": int(y.numel() * y.element_size()), "ms_per_step": e2e_ms,
               "pipeline": "copy-in, oq_qlinear and copy-out on three streams, two buffers deep",
               "schedule": e2e_schedule}

    peaks = measured_peaks()
    # the fp8 variant's contraction peak: the measured bf16 peak times the
    # nominal e4m3 / bf16 dense ratio (4.5 / 2.25 PFLOP/s)
    mma_peak = peaks["bf16_tflops"] * (2.0 if args.fp8 else 1.0)
    peak_note = peaks["source"] + (" bf16 (burst) x nominal fp8/bf16 ratio 2" if args.fp8 else " (burst)")
    flops = 2.0 * w.M * w.N * w.d
    gemm_tflops = flops / (ms_gemm * 1e-3) / 1e12
    step_tflops = flops / (ms * 1e-3) / 1e12
    rb = rpbh_bytes(w, schedule, args.fp8)
    rpbh_gbs = rb / (ms_rpbh * 1e-3) / 1e9
    gemm_key = ("qgemm_values" if schedule == "values" else "qgemm") + ("_fp8" if args.fp8 else "")
    rpbh_key = "rpbh_quant" + (("_values_fp8" if args.fp8 else "_values") if schedule == "values" else "")
    out = {
        "metric": METRIC, "value": job_throughput(world, w.M, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if args.fp8 else "bf16", "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "d": w.d, "N": w.N, "h": w.h, "bits_w": w.bits_w,
                   "bits_a": w.bits_a, "x_dtype": w.x_dtype, "tokens_per_gpu": w.M, "global_batch": world * w.M,
                   "parallelism": f"dp{world} (replicated packed W, no collective)", "schedule": schedule,
                   "l2": "flushed (256 MB write) before every timed step, outside the events"},
        "tflops": step_tflops,
        "breakdown": {"rpbh_quant_ms": ms_rpbh, "qgemm_ms": ms_gemm, "qgemm_tflops": gemm_tflops,
                      "rpbh_quant_gbs": rpbh_gbs},
        "roofline": {"bound": "tensor", "kernel": gemm_key, "achieved": gemm_tflops,
                     "peak": mma_peak, "unit": "TFLOP/s", "frac": gemm_tflops / mma_peak,
                     "traffic": committed_traffic(gemm_key, w.name), "peak_source": peak_note,
                     "algorithmic": f"2*M*N*d = {flops:.4g} flop per launch"},
        "roofline_rpbh": {"bound": "hbm", "kernel": rpbh_key, "achieved": rpbh_gbs, "peak": peaks["hbm_gbs"],
                          "unit": "GB/s", "frac": rpbh_gbs / peaks["hbm_gbs"],
                          "traffic": committed_traffic(rpbh_key, w.name),
                          "algorithmic": f"M*(d*in_bytes + {'values' if schedule == 'values' else 'packed'} + 4) = "
                                         f"{rb} B per launch"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok_s, rows, dt, thr = cpu_oracle_sample(w, x_cpu, w_idx.cpu(), w_r.cpu(), args.cpu_seconds, w.M)
        out["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                               "sample": f"{rows} tokens of {w.name}: rotate+quantise each row, then its full "
                                         f"{w.N}-wide output row ({dt:.1f} s)"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_ablation(args):
    """The page's rotation ablation on one GPU: the fused rotate+quantise
    kernel with the RPBH plan and with the Block-RHT plan (no permutation),
    the rotation alone for both (oq_rpbh_apply), and a dense Haar rotation
    (a cuBLAS bf16 GEMM against a random orthogonal d x d matrix).  Median
    device time per call over --steps calls, L2 flushed before each."""
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
    plans = {"rpbh": B.rpbh_plan(w.d, w.h, w.plan_seed),
             "block_rht": B.rotation_plan(w.d, w.h, w.plan_seed, B.OQ_ROT_BLOCK_RHT)}
    packed = w.d if w.bits_a == 6 else w.d * w.bits_a // 8
    a_idx = torch.empty((w.M, packed), dtype=torch.uint8, device=dev)
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
    calls = {
        "rpbh_quant": lambda: B.quantize_acts(plans["rpbh"], cb_a, x, a_idx, s, stream=stream),
        "block_rht_quant": lambda: B.quantize_acts(plans["block_rht"], cb_a, x, a_idx, s, stream=stream),
        "rpbh_rotate": lambda: B.rpbh_apply(plans["rpbh"], x, x_rot, s, stream=stream),
        "block_rht_rotate": lambda: B.rpbh_apply(plans["block_rht"], x, x_rot, s, stream=stream),
        "haar_rotate_cublas": lambda: torch.matmul(xb, haar_t, out=y_haar),
    }
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
        "workload": w.name, "M": w.M, "d": w.d, "h": w.h, "bits_a": w.bits_a, "steps": args.steps,
        "ms": ms,
        "ratios": {
            "rpbh_over_block_rht_quant": ms["rpbh_quant"] / ms["block_rht_quant"],
            "rpbh_over_block_rht_rotate": ms["rpbh_rotate"] / ms["block_rht_rotate"],
            "haar_over_rpbh_rotate": ms["haar_rotate_cublas"] / ms["rpbh_rotate"],
            "haar_over_rpbh_quant": ms["haar_rotate_cublas"] / ms["rpbh_quant"],
        },
        "note": "rotate = oq_rpbh_apply (fp32 x' and norms out); quant = the fused rotate+split+quantise kernel; "
                "haar = bf16 x @ Q^T with a Haar-random Q, bf16 out (cuBLAS); L2 flushed before every call",
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.ablation:
        run_ablation(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
