#!/usr/bin/env python
"""Benchmark of the spectral-split W4A4 linear layer on one B200 per rank.

Workload (``layer_4096``): W bf16 4096 x 4096 with a planted spectrum
sigma_i = 8/i (i <= 256) + N(0, 0.02^2) noise, X bf16 8192 x 4096 N(0, 1);
one step = metis_split of W (k=64, p=16, one power iteration, Gaussian
sketch, NVFP4 residual along K, FP4 factors) + metis_quantize_fp4 of X along K
(NVFP4) + metis_linear_fwd Y = X W (FP4 GEMM with the rank-64 update fused,
bf16 output).  Inputs are synthetic and seeded (no dataset).

Metric: effective FP4 split-linear TFLOPS = 2 M N K (the dense product the
layer replaces) / step time, plus the split + quantize time per layer.
Timing: CUDA events on the launching stream around a CUDA-graph replay of the
step, L2 (126 MB) flushed with a 512 MB write before every timed step, W >= 3
warm-up steps, max over ranks.  With torchrun and N GPUs every rank runs the
same layer independently (replicas: the path has no cross-GPU exchange), and
``value`` is the work of all ranks over the slowest rank's time.

``--impl reference`` times the CPU oracle (numpy) on a bounded sample of the
same workload instead: the oracle is the only reference implementation this
path has.
"""
import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M, K, N = 8192, 4096, 4096
RANK_K, OVERSAMPLE, POWER_ITERS, SEED = 64, 16, 1, 0
FLOPS = 2.0 * M * N * K
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the plain-operand FP4 GEMM, from one ncu capture of the current kernel; to
# be set to None whenever the kernel changes after that capture.
GEMM_NCU_DRAM_BYTES = 34.673920e6 + 18.095104e6
METRIC = "FP4 split-linear eff. TFLOPS & % of FP4 peak; split+quantize us/layer"
CONFIG = {"workload": "layer_4096: W bf16 4096x4096 planted spectrum + X bf16 8192x4096, "
                      "split k=64 p=16 q=1 Gaussian, NVFP4, forward",
          "M": M, "K": K, "N": N, "k": RANK_K, "p": OVERSAMPLE, "power_iters": POWER_ITERS,
          "fmt": "nvfp4", "l2": "flushed (512 MB write) before every timed step"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--compensate", action="store_true",
                    help="the split forms the error-compensated residual A - deq(U_q) S deq(V_q)^T")
    ap.add_argument("--composite", action="store_true",
                    help="measure the mean + spectral composite split of the Averis-shaped activation instead")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="run this many eager steps (no graphs, no timing) and exit: the command profiled by ncu")
    return ap.parse_args()


# --------------------------------------------------------------------------
# distributed plumbing (replicas; barriers and a max-reduction only)
# --------------------------------------------------------------------------

def dist_backend():
    """The process-group backend: METIS_DIST_BACKEND ("nccl" or "gloo") when
    set, else NCCL where CUDA is available and gloo otherwise.  gloo keeps
    the timing reduction on host tensors."""
    import torch
    b = os.environ.get("METIS_DIST_BACKEND", "").strip().lower()
    if b:
        if b not in ("nccl", "gloo"):
            raise ValueError(f"METIS_DIST_BACKEND must be nccl or gloo, not {b!r}")
        return b
    return "nccl" if torch.cuda.is_available() else "gloo"


def dist_init():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = dist_backend()
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    """SM clock, its maximum and the clock-event (throttle) reasons, sampled
    during the timed region.  NVML is read from a thread every 2 ms (a timed
    region of a few tens of milliseconds still gets samples); where NVML is
    not importable, `nvidia-smi -lms 50` runs instead, started before the
    region.  Nothing here changes a setting of the GPU."""

    REASONS = (("hw_slowdown", 8), ("hw_thermal_slowdown", 64), ("sw_thermal_slowdown", 32),
               ("sw_power_cap", 4), ("hw_power_brake_slowdown", 128))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.thread = None
        self.proc = None
        self.path = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.index).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop_evt = threading.Event()

            def run():
                while not self.stop_evt.is_set():
                    try:
                        self.rows.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                          int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        pass
                    self.stop_evt.wait(0.002)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            self.source = "nvml (2 ms)"
            return
        except Exception:
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()
            while os.path.getsize(self.path) == 0 and time.time() - t0 < 5.0:
                time.sleep(0.01)   # the first sample lands before the timed region starts
            self.source = "nvidia-smi (50 ms)"
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            if not self.rows:
                return None
            sm = [r[0] for r in self.rows]
            loaded = [v for v in sm if v > 0.5 * self.smax] or sm
            reasons = sorted({name for _, bits in self.rows for name, bit in self.REASONS if bits & bit})
            return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": self.smax, "reasons": reasons,
                    "samples": len(self.rows), "source": self.source}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        loaded = [v for v in sm if v > 0.5 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "source": self.source}


# --------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------

ORACLE_ROWS = 1024   # rows of X in the oracle's sample (cpu_baseline and the reference arm alike)


def oracle_sample(data, rows=ORACLE_ROWS):
    """The oracle's whole step on a bounded sample, timed in two parts.

    Row-independent (done once per step whatever M is): the split of W, the
    FP4 quantization of its residual and factors, and the dense float64 value
    of W's operand (dequantized and assembled).  Row-proportional: the FP4
    quantization of X and the float64 product, on the first `rows` rows of X;
    rows are independent, so this part scales by M / rows.

    Returns (seconds extrapolated to the full step, seconds spent, description)."""
    from oracle import fp4, gemm, split
    t0 = time.perf_counter()
    W = data["W"].f64()
    r = split.split(W, RANK_K, OVERSAMPLE, POWER_ITERS, SEED)
    Rq = fp4.quantize(r["R"].astype(np.float32), "nv", 0)
    Uq = fp4.quantize(r["U"].astype(np.float32), "nv", 0)
    Vq = fp4.quantize(r["V"].astype(np.float32), "nv", 0)
    Wd = gemm.dense_right(gemm.Operand(Rq, RANK_K, Uq, Vq, r["S"]))
    t_fixed = time.perf_counter() - t0
    t1 = time.perf_counter()
    xq = fp4.quantize(data["X"].f32()[:rows], "nv", 1)
    gemm.dense_left(gemm.Operand(xq)) @ Wd
    t_rows = time.perf_counter() - t1
    full = t_fixed + t_rows * (M / rows)
    desc = (f"split of W, its FP4 outputs and W's dense operand once; X quantize + product on {rows} of "
            f"{M} rows, that part scaled x{M // rows}")
    return full, t_fixed + t_rows, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank, world):
    """The oracle (numpy, host cores) on the same sample as cpu_baseline.
    ms_per_step is the wall time of one sampled step as it ran; the metric
    divides the full step's flops by the time extrapolated to the full step
    (reported as full_step_ms_extrapolated)."""
    if rank != 0:
        return
    from spectral_domain_quantization_b200 import inputs
    data = inputs.make("layer_4096")
    for _ in range(args.warmup):
        oracle_sample(data)
    full, spent = [], []
    desc = ""
    for _ in range(args.steps):
        f, t, desc = oracle_sample(data)
        full.append(f)
        spent.append(t)
    full_s = float(np.mean(full))
    value = FLOPS / full_s / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(spent)) * 1e3,
            "full_step_ms_extrapolated": full_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": CONFIG,
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": "TFLOPS", "cores": cores,
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# the GPU path
# --------------------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def run_ours(args, rank, world, local):
    import torch
    from spectral_domain_quantization_b200 import api, inputs

    assert torch.cuda.is_available(), "bench needs a GPU"
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if not api.lib().metis_device_supported():
        raise RuntimeError("metis needs an sm_100 (B200) device")
    data = inputs.make("layer_4096")
    w_host = torch.from_numpy(data["W"].data.view(np.int16)).view(torch.bfloat16).pin_memory()
    x_host = torch.from_numpy(data["X"].data.view(np.int16)).view(torch.bfloat16).pin_memory()
    W = w_host.to(dev)
    X = x_host.to(dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def make_step(Wb, Xb, Yb):
        def split_w():
            return api.split(Wb, RANK_K, OVERSAMPLE, POWER_ITERS, SEED, "nv", rows=False, cols=True, factors=True,
                             compensate=args.compensate, dev_status=status)

        def quant_x():
            return api.quantize_fp4(Xb, "nv", 1)

        def step():
            # X's quantization does not depend on W's split: it runs on a second
            # stream while the split's single-CTA phases leave most SMs idle
            main = torch.cuda.current_stream()
            side.wait_stream(main)
            with torch.cuda.stream(side):
                xq = quant_x()
            s = split_w()
            main.wait_stream(side)
            api.linear_fwd(api.Operand(xq), s.operand("right"), M, N, K, Y=Yb, dev_status=status)

        return split_w, quant_x, step

    side = torch.cuda.Stream(device=dev)
    split_w, quant_x, step = make_step(W, X, Y)

    def capture(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g

    def time_graph(g, steps, warmup):
        for _ in range(warmup):
            flush.fill_(1)
            g.replay()
        torch.cuda.synchronize()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush.fill_(1)
            starts[i].record()
            g.replay()
            ends[i].record()
        torch.cuda.synchronize()
        return float(np.mean([s.elapsed_time(e) for s, e in zip(starts, ends)]))

    # --- the step, as one CUDA graph
    g_step = capture(step)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")

    # kernels of this library launched by one step
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize()
    launches = sum(1 for e in prof.events() if e.device_type.name == "CUDA" and "metis" in e.name)

    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    ms = time_graph(g_step, args.steps, args.warmup)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = reduce_max(ms, world)

    # --- phase breakdown (same flush policy)
    g_split = capture(split_w)
    ms_split = time_graph(g_split, args.steps, 3)
    g_quant = capture(quant_x)
    ms_quant = time_graph(g_quant, args.steps, 3)
    s = split_w()
    xq = quant_x()
    g_gemm = capture(lambda: api.linear_fwd(api.Operand(xq), s.operand("right"), M, N, K, Y=Y, dev_status=status))
    ms_gemm = time_graph(g_gemm, args.steps, 3)
    # the FP4 GEMM kernel alone (plain operands: one launch of the kernel)
    rq = s.R_cols
    g_plain = capture(lambda: api.linear_fwd(api.Operand(xq), api.Operand(rq), M, N, K, Y=Y, dev_status=status))
    ms_plain = time_graph(g_plain, args.steps, 3)

    # --- end to end through host buffers: every step copies its inputs from
    # pinned host memory and its output back; two buffer sets let step i+1's
    # uploads and step i-1's download overlap step i's compute (copy engines
    # in both directions and the SMs all busy, as a pipelined caller would)
    e2e = None
    if not args.no_e2e:
        W1, X1 = torch.empty_like(W), torch.empty_like(X)
        Y1 = torch.empty_like(Y)
        g_step1 = capture(make_step(W1, X1, Y1)[2])
        sets = [(W, X, Y, g_step), (W1, X1, Y1, g_step1)]
        y_host = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        comp = torch.cuda.current_stream()
        h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        up = [torch.cuda.Event() for _ in range(2)]
        ran = [torch.cuda.Event() for _ in range(2)]
        down = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i & 1
            Wb, Xb, Yb, gb = sets[b]
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(ran[b])        # set b's inputs are no longer read
                Wb.copy_(w_host, non_blocking=True)
                Xb.copy_(x_host, non_blocking=True)
                up[b].record(h2d)
            comp.wait_event(up[b])
            if i >= 2:
                comp.wait_event(down[b])          # set b's output has been copied out
            gb.replay()
            ran[b].record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ran[b])
                y_host[b].copy_(Yb, non_blocking=True)
                down[b].record(d2h)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        h2d.wait_stream(comp)
        for i in range(args.steps):
            e2e_step(i)
        comp.wait_stream(d2h)
        e1.record(comp)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, world)
        e2e = {"value": world * FLOPS / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
               "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(w_host.numel() * 2 + x_host.numel() * 2),
               "d2h_bytes_per_step": int(M * N * 2),
               "pipelining": "double-buffered: uploads, compute and download of consecutive steps overlap"}
        del g_step1

    hbm, bf16_tf, peak_kind = measured_peaks()
    fp4_peak = 4.0 * bf16_tf   # nominal dense FP4 / bf16 ratio on B200 (9 / 2.25 PFLOP/s)
    achieved = FLOPS / (ms_plain * 1e-3) / 1e12
    value = world * FLOPS / (ms * 1e-3) / 1e12

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        reps = []
        desc = ""
        t_end = time.time() + 20
        while time.time() < t_end or not reps:
            t, _, desc = oracle_sample(data)
            reps.append(t)
        cpu = {"value": FLOPS / float(np.mean(reps)) / 1e12, "unit": "TFLOPS", "cores": blas_threads(),
               "kind": "oracle", "sample": desc + f"; {len(reps)} repetitions",
               "full_step_ms_extrapolated": float(np.mean(reps)) * 1e3}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp4 (e2m1, nvfp4 scales; fp32 accumulate)", "data": "synthetic",
            "config": dict(CONFIG, residual="error-compensated: A - deq(U_q) S deq(V_q)^T") if args.compensate
            else CONFIG,
            "frac_of_fp4_peak": value / world / fp4_peak,
            "split_quantize_us_per_layer": (ms_split + ms_quant) * 1e3,
            "breakdown_us": {"split_W": ms_split * 1e3, "quantize_X": ms_quant * 1e3,
                             "linear_fwd": ms_gemm * 1e3, "fp4_gemm_kernel": ms_plain * 1e3},
            "roofline": {"kernel": "gemm_fp4_kernel<256,4,1> (8192x4096x4096 NVFP4)", "bound": "tensor",
                         "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                         "peak_source": f"{peak_kind} bf16 {bf16_tf} TFLOP/s x 4 (nominal FP4/bf16 ratio)",
                         "traffic": GEMM_NCU_DRAM_BYTES},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    # release graphs before the process group goes away
    del g_step, g_split, g_quant, g_gemm, g_plain


def run_profile(args, local):
    """The step, eagerly and untimed: a short launch list for profilers."""
    import torch
    from spectral_domain_quantization_b200 import api, inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    data = inputs.make("layer_4096")
    W = torch.from_numpy(data["W"].data.view(np.int16)).view(torch.bfloat16).to(dev)
    X = torch.from_numpy(data["X"].data.view(np.int16)).view(torch.bfloat16).to(dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(args.profile_steps):
        s = api.split(W, RANK_K, OVERSAMPLE, POWER_ITERS, SEED, "nv", rows=False, cols=True, factors=True,
                      dev_status=status)
        xq = api.quantize_fp4(X, "nv", 1)
        api.linear_fwd(api.Operand(xq), s.operand("right"), M, N, K, Y=Y, dev_status=status)
    torch.cuda.synchronize()
    print(json.dumps({"profile_steps": args.profile_steps, "dev_status": int(status.item())}), flush=True)


def run_composite(args, local):
    """The mean + spectral composite: averis_split of an activation with a
    column mean (X bf16 32768 x 4096 = 1 mu^T + Z), the spectral split of its
    float32 mean-free residual (k = 64, p = 16, q = 1), the rank-65 FP4
    factors, then Y = X W with the composite X and a plain NVFP4 W.  Eager
    calls timed with CUDA events on the current stream, L2 flushed before
    every step; one JSON line."""
    import torch
    from spectral_domain_quantization_b200 import api, inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    data = inputs.make("averis_32768", keys=("X", "W"))
    c = data["cfg"]
    Mx, Kx, Nx = c["M"], c["K"], c["N"]
    X = torch.from_numpy(data["X"].data.view(np.int16)).view(torch.bfloat16).to(dev)
    W = torch.from_numpy(data["W"].data.view(np.int16)).view(torch.bfloat16).to(dev)
    qw = api.quantize_fp4(W, "nv", 0)                       # outer N, blocks along K
    Y = torch.empty((Mx, Nx), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.int16, device=dev)
    t_split, t_fwd = [], []
    for i in range(args.warmup + args.steps):
        flush.fill_(1)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        comp = api.composite_split(X, RANK_K, OVERSAMPLE, POWER_ITERS, SEED, "nv", rows=True, cols=False,
                                   dev_status=status)
        e1.record()
        api.linear_fwd(comp.operand("left"), api.Operand(qw), Mx, Nx, Kx, Y=Y, dev_status=status)
        e2.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            t_split.append(e0.elapsed_time(e1))
            t_fwd.append(e1.elapsed_time(e2))
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    split_ms, fwd_ms = float(np.mean(t_split)), float(np.mean(t_fwd))
    flops = 2.0 * Mx * Nx * Kx
    line = {"metric": "mean + spectral composite split us/layer; composite forward eff. TFLOPS",
            "value": split_ms * 1e3, "unit": "us", "higher_is_better": False, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "dtype": "fp4 (e2m1, nvfp4 scales; fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": f"averis_32768 activation X bf16 {Mx}x{Kx} = 1 mu^T + Z; composite split "
                                   f"k={RANK_K} p={OVERSAMPLE} q={POWER_ITERS} (rank {RANK_K + 1} with the mean), "
                                   f"NVFP4; Y = X W with W bf16 {Kx}x{Nx} plain NVFP4",
                       "timing": "eager calls, CUDA events, L2 flushed (512 MB write) before every step"},
            "breakdown_us": {"composite_split": split_ms * 1e3, "forward_product": fwd_ms * 1e3},
            "forward_tflops": flops / (fwd_ms * 1e-3) / 1e12}
    if not args.no_cpu_baseline:
        from oracle import composite
        rows = 2048
        x32 = data["X"].f32()[:rows]
        t0 = time.perf_counter()
        composite.split(x32, RANK_K, OVERSAMPLE, POWER_ITERS, SEED)
        dt = (time.perf_counter() - t0) * (Mx / rows)
        line["cpu_baseline"] = {"value": dt * 1e6, "unit": "us", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"composite split of the first {rows} of {Mx} rows, scaled x{Mx // rows}"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.profile_steps > 0:
        run_profile(args, int(os.environ.get("LOCAL_RANK", "0")))
        return
    if args.composite:
        # a single-GPU measurement: under a multi-process launch only rank 0 runs it
        if int(os.environ.get("RANK", "0")) == 0:
            run_composite(args, int(os.environ.get("LOCAL_RANK", "0")))
        return
    rank, world, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
