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
# algorithmic bytes of the split of W (four passes of the range finder and two
# residual passes over W, the NVFP4 copy of R, the float32 factors and their
# FP4 copies) and of X's NVFP4 quantization (the amax pass and the quantizing
# pass over X, its codes and scales): each byte the method must move, once
# per pass
SPLIT_W_BYTES = (6 * K * N * 2 + (K * N // 2 + K * N // 16) + (K + N) * RANK_K * 4
                 + (K + N) * RANK_K // 2 + (K + N) * RANK_K // 16)
QUANT_X_BYTES = 2 * M * K * 2 + M * K // 2 + M * K // 16
FLOPS = 2.0 * M * N * K
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the plain-operand FP4 GEMM, from one ncu capture of the current kernel; None
# whenever the kernel changed after that capture (the last capture, 50.7 MB,
# predates the separate scale barrier).
GEMM_NCU_DRAM_BYTES = None
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
    ap.add_argument("--workload", default="layer_4096",
                    choices=["layer_4096", "averis_32768", "llama3_8b_mlp", "sampled_65536"],
                    help="the timed step: the single layer (default) or another synthetic workload")
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
            "hbm": {name: {"algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (t * 1e-3) / 1e9,
                           "peak_gbs": hbm, "frac": nbytes / (t * 1e-3) / 1e9 / hbm, "peak_source": peak_kind}
                    for name, nbytes, t in (("split_W", SPLIT_W_BYTES, ms_split), ("quantize_X", QUANT_X_BYTES, ms_quant))},
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


# --------------------------------------------------------------------------
# the other synthetic workloads (--workload): one step each, the same timing
# rules; the split / quantize phase is also reported against the HBM peak
# with its algorithmic bytes (each input byte read and each output byte
# written once per pass the method needs)
# --------------------------------------------------------------------------

def _fp4_bytes(rows, cols, fmt):
    """codes + scale bytes of one FP4 copy of a rows x cols matrix."""
    return rows * cols // 2 + rows * cols // (32 if fmt == "mx" else 16)


class AverisWorkload:
    """averis_32768: X bf16 32768 x 4096 = 1 mu^T + Z (0.1 % outliers), W bf16
    4096 x 4096, dY bf16 32768 x 4096.  Step: the Averis split of X and of dY
    (NVFP4, both block axes), W quantized along K and along N, then Y = X W,
    dX = dY W^T and dW = X^T dY (bf16 outputs)."""

    name = "averis_32768"

    def __init__(self, dev):
        import torch
        from spectral_domain_quantization_b200 import api, inputs
        self.api = api
        d = inputs.make("averis_32768")
        c = d["cfg"]
        self.M, self.K, self.N = c["M"], c["K"], c["N"]
        self.host = {k: _pinned_bf16(d[k]) for k in ("X", "W", "dY")}
        self.dev = {k: v.to(dev) for k, v in self.host.items()}
        self.Y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty((self.M, self.K), dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty((self.K, self.N), dtype=torch.bfloat16, device=dev)
        self.data = d
        M, K, N = self.M, self.K, self.N
        self.flops = 3 * 2.0 * M * N * K
        # X and dY: two reads (the column sums, then the residual pass) and
        # two FP4 copies each; W: amax and quantize reads per axis, two copies
        self.split_bytes = (2 * (2 * M * K * 2 + 2 * _fp4_bytes(M, K, "nv"))
                            + 2 * (2 * K * N * 2 + _fp4_bytes(K, N, "nv")))
        self.config = {"workload": "averis_32768: X bf16 32768x4096 = 1 mu^T + Z, dY bf16 32768x4096, W bf16 "
                                   "4096x4096; Averis split of X and dY, W plain, NVFP4; forward, dX, dW",
                       "M": M, "K": K, "N": N, "fmt": "nvfp4"}
        self.ops = None

    def split(self):
        api, d = self.api, self.dev
        self.ops = (api.averis_split(d["X"], "nv"), api.averis_split(d["dY"], "nv"),
                    api.quantize_fp4(d["W"], "nv", 0), api.quantize_fp4(d["W"], "nv", 1))

    def products(self):
        api = self.api
        ax, ady, qw_k, qw_n = self.ops
        api.linear_fwd(ax.left(), api.Operand(qw_k), self.M, self.N, self.K, Y=self.Y)
        api.linear_bwd(ady.left(), api.Operand(qw_n), ax.left_t(), ady.right_m(), self.M, self.N, self.K,
                       out_dtype=self.Y.dtype, dX=self.dX, dW=self.dW)

    def plain(self):
        """the largest product with plain operands: one launch of the FP4 GEMM kernel"""
        api = self.api
        ax, _, qw_k, _ = self.ops
        api.linear_fwd(api.Operand(ax.R_rows), api.Operand(qw_k), self.M, self.N, self.K, Y=self.Y)
        return 2.0 * self.M * self.N * self.K, f"gemm_fp4 ({self.M}x{self.N}x{self.K} NVFP4)"

    def outputs(self):
        return [self.Y, self.dX, self.dW]

    def oracle_sample(self, rows=256):
        from oracle import averis, fp4, gemm
        d = self.data
        t0 = time.perf_counter()
        out = []
        for key in ("X", "dY"):
            x = d[key].f64()
            mu, _ = averis.split(x)               # the column mean needs every row
            out.append((x, mu))
        W = d["W"].f32()
        qk, qn = fp4.quantize(W, "nv", 0), fp4.quantize(W, "nv", 1)
        wk, wn = gemm.dense_right(gemm.Operand(qk)), gemm.dense_right(gemm.Operand(qn)).T
        t_fixed = time.perf_counter() - t0
        t1 = time.perf_counter()
        (x, mu), (dy, nu) = out
        rx = np.float32(x[:rows] - mu)
        rdy = np.float32(dy[:rows] - nu)
        xq = fp4.quantize(rx, "nv", 1)
        dyq = fp4.quantize(rdy, "nv", 1)
        (xq.dequantize() + mu[None, :]) @ wk
        (dyq.dequantize() + nu[None, :]) @ wn.T
        # dW = X^T dY over the sampled rows (its share of the contraction)
        fp4.quantize(rx, "nv", 0).dequantize() @ fp4.quantize(rdy, "nv", 0).dequantize().T
        t_rows = time.perf_counter() - t1
        full = t_fixed + t_rows * (self.M / rows)
        return full, t_fixed + t_rows, (f"column means of X and dY, W's two FP4 copies once; residuals, their FP4 "
                                        f"copies and the three products on {rows} of {self.M} rows, scaled "
                                        f"x{self.M // rows}")


class LlamaMlpWorkload:
    """llama3_8b_mlp (gate projection): W bf16 4096 x 14336 (planted), X bf16
    16384 x 4096, dY bf16 16384 x 14336.  Step: the spectral split of W, X and
    dY (k = 64, p = 16, q = 1, NVFP4, residuals along both axes, FP4 factors),
    then Y = X W, dX = dY W^T and dW = X^T dY (bf16 outputs)."""

    name = "llama3_8b_mlp"

    def __init__(self, dev):
        import torch
        from spectral_domain_quantization_b200 import api, inputs
        self.api = api
        d = inputs.make("llama3_8b_mlp", keys=("W", "X", "dY"))
        c = d["cfg"]
        self.c = c
        self.M, self.K, self.N, self.k = c["M"], c["K"], c["N"], c["k"]
        self.host = {k: _pinned_bf16(d[k]) for k in ("W", "X", "dY")}
        self.dev = {k: v.to(dev) for k, v in self.host.items()}
        self.Y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty((self.M, self.K), dtype=torch.bfloat16, device=dev)
        self.dW = torch.empty((self.K, self.N), dtype=torch.bfloat16, device=dev)
        self.data = d
        M, K, N, k = self.M, self.K, self.N, self.k
        self.flops = 3 * 2.0 * M * N * K

        def split_bytes(m, n):   # four sketch passes and two residual passes, two FP4 copies, the factors
            return 6 * m * n * 2 + 2 * _fp4_bytes(m, n, "nv") + (m + n) * k * 4 + _fp4_bytes(k, m + n, "nv")
        self.split_bytes = split_bytes(K, N) + split_bytes(M, K) + split_bytes(M, N)
        self.config = {"workload": "llama3_8b_mlp gate projection: W bf16 4096x14336 planted spectrum, X bf16 "
                                   "16384x4096, dY bf16 16384x14336; split k=64 p=16 q=1 Gaussian of W, X, dY, "
                                   "NVFP4; forward, dX, dW",
                       "M": M, "K": K, "N": N, "k": k, "p": c["p"], "power_iters": c["q"], "fmt": "nvfp4"}
        self.ops = None
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(3)]

    def split(self):
        # the three splits are independent: each runs on its own stream, so
        # one split's single-CTA factorisations overlap the others' HBM passes
        import torch
        api, d, c = self.api, self.dev, self.c
        args = (self.k, c["p"], c["q"], c["sketch_seed"], "nv")
        main = torch.cuda.current_stream()
        ops = []
        for key, s in zip(("W", "X", "dY"), self.streams):
            s.wait_stream(main)
            with torch.cuda.stream(s):
                ops.append(api.split(d[key], *args, rows=True, cols=True))
        for s in self.streams:
            main.wait_stream(s)
        self.ops = tuple(ops)

    def products(self):
        api = self.api
        Ws, Xs, Ds = self.ops
        k = self.k
        api.linear_fwd(Xs.operand("left"), Ws.operand("right"), self.M, self.N, self.K, Y=self.Y)
        api.linear_bwd(Ds.operand("left"), api.Operand(Ws.R_rows, k, Ws.V_q, Ws.U_q, Ws.S),
                       api.Operand(Xs.R_cols, k, Xs.U_q, Xs.V_q, Xs.S), Ds.operand("right"), self.M, self.N,
                       self.K, out_dtype=self.Y.dtype, dX=self.dX, dW=self.dW)

    def plain(self):
        api = self.api
        Ws, Xs, _ = self.ops
        api.linear_fwd(api.Operand(Xs.R_rows), api.Operand(Ws.R_cols), self.M, self.N, self.K, Y=self.Y)
        return 2.0 * self.M * self.N * self.K, f"gemm_fp4 ({self.M}x{self.N}x{self.K} NVFP4)"

    def outputs(self):
        return [self.Y, self.dX, self.dW]

    def oracle_sample(self, rows=64):
        from oracle import fp4, gemm, split
        d, c, k = self.data, self.c, self.k
        t0 = time.perf_counter()
        res = {}
        for key in ("W", "X", "dY"):
            res[key] = split.split(d[key].f64(), k, c["p"], c["q"], c["sketch_seed"])
        q = lambda a, axis: fp4.quantize(np.float32(a), "nv", axis)
        w, x, dy = res["W"], res["X"], res["dY"]
        # W's two dense operands do not depend on the rows
        wr = gemm.dense_right(gemm.Operand(q(w["R"], 0), k, q(w["U"], 0), q(w["V"], 0), w["S"]))
        wt = gemm.dense_right(gemm.Operand(q(w["R"], 1), k, q(w["V"], 0), q(w["U"], 0), w["S"]))
        t_split = time.perf_counter() - t0
        t1 = time.perf_counter()
        # the rows' share of each product: forward and dX on `rows` rows of
        # X / dY, dW on `rows` rows of the contraction over M
        xl = gemm.Operand(q(x["R"][:rows], 1), k, q(x["V"], 0), q(x["U"][:rows], 0), x["S"])
        gemm.dense_left(xl) @ wr
        dl = gemm.Operand(q(dy["R"][:rows], 1), k, q(dy["V"], 0), q(dy["U"][:rows], 0), dy["S"])
        gemm.dense_left(dl) @ wt
        xt = gemm.dense_left(gemm.Operand(q(x["R"][:rows], 0), k, q(x["U"][:rows], 0), q(x["V"], 0), x["S"]))
        dr = gemm.dense_right(gemm.Operand(q(dy["R"][:rows], 0), k, q(dy["U"][:rows], 0), q(dy["V"], 0), dy["S"]))
        xt @ dr
        t_rows = time.perf_counter() - t1
        full = t_split + t_rows * (self.M / rows)
        return full, t_split + t_rows, (f"splits of W, X and dY and W's dense operands once; FP4 operands and the "
                                        f"three products on {rows} of {self.M} rows, scaled x{self.M // rows}")


class SampledWorkload:
    """sampled_65536: A bf16 65536 x 4096 with a planted rank-32 spike, W bf16
    4096 x 4096.  Step: the sampled split of A (2048 rows, sparse-sign sketch
    with 4 nonzeros, k = 32, p = 16, q = 0, MXFP4, residual along K), W
    quantized along K, then Y = A W (bf16 output)."""

    name = "sampled_65536"

    def __init__(self, dev):
        import torch
        from spectral_domain_quantization_b200 import api, inputs
        self.api = api
        d = inputs.make("sampled_65536")
        c = d["cfg"]
        self.c = c
        self.M, self.K, self.N, self.k = c["M"], c["K"], c["N"], c["k"]
        self.host = {k: _pinned_bf16(d[k]) for k in ("A", "W")}
        self.dev = {k: v.to(dev) for k, v in self.host.items()}
        self.Y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=dev)
        self.data = d
        M, K, N, k, s = self.M, self.K, self.N, self.k, c["sample_rows"]
        self.flops = 2.0 * M * N * K
        # gather s rows, two passes over them, one pass over A (P = A V_s, the
        # residual and its FP4 copy), the W copy (one read, codes and scales)
        self.split_bytes = (s * K * 2 * 3 + M * K * 2 + _fp4_bytes(M, K, "mx") + M * k * 4 * 2
                            + K * N * 2 + _fp4_bytes(K, N, "mx"))
        self.config = {"workload": "sampled_65536: A bf16 65536x4096 planted rank-32 spike, W bf16 4096x4096; "
                                   "2048 sampled rows, sparse-sign sketch (4 nnz), k=32 p=16 q=0, MXFP4; forward",
                       "M": M, "K": K, "N": N, "k": k, "p": c["p"], "sample_rows": s, "fmt": "mxfp4"}
        self.ops = None
        self.side = torch.cuda.Stream(device=dev)

    def split(self):
        # W's quantization does not depend on A's split: it runs on a second stream
        import torch
        api, d, c = self.api, self.dev, self.c
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            qw = api.quantize_fp4(d["W"], "mx", 0)
        As = api.split(d["A"], self.k, c["p"], 0, c["sketch_seed"], "mx", sketch="sparse_sign", nnz=4,
                       sample_rows=c["sample_rows"], rows=True, cols=False)
        main.wait_stream(self.side)
        self.ops = (As, qw)

    def products(self):
        api = self.api
        As, qw = self.ops
        api.linear_fwd(As.operand("left"), api.Operand(qw), self.M, self.N, self.K, Y=self.Y)

    def plain(self):
        api = self.api
        As, qw = self.ops
        api.linear_fwd(api.Operand(As.R_rows), api.Operand(qw), self.M, self.N, self.K, Y=self.Y)
        return 2.0 * self.M * self.N * self.K, f"gemm_fp4 ({self.M}x{self.N}x{self.K} MXFP4)"

    def outputs(self):
        return [self.Y]

    def oracle_sample(self, rows=512):
        from oracle import fp4, gemm, split
        d, c, k = self.data, self.c, self.k
        t0 = time.perf_counter()
        A = d["A"].f64()
        r = split.split(A, k, c["p"], 0, c["sketch_seed"], kind="sparse_sign", nnz=4, sample_rows=c["sample_rows"])
        wr = gemm.dense_right(gemm.Operand(fp4.quantize(d["W"].f32(), "mx", 0)))
        t_fixed = time.perf_counter() - t0
        t1 = time.perf_counter()
        q = lambda a, axis: fp4.quantize(np.float32(a), "mx", axis)
        left = gemm.Operand(q(r["R"][:rows], 1), k, q(r["V"], 0), q(r["U"][:rows], 0), r["S"])
        gemm.dense_left(left) @ wr
        t_rows = time.perf_counter() - t1
        full = t_fixed + t_rows * (self.M / rows)
        return full, t_fixed + t_rows, (f"sampled split of A and W's FP4 copy once; the residual rows' FP4 copy and "
                                        f"the product on {rows} of {self.M} rows, scaled x{self.M // rows}")


WORKLOADS = {"averis_32768": AverisWorkload, "llama3_8b_mlp": LlamaMlpWorkload,
             "sampled_65536": SampledWorkload}


def _pinned_bf16(mat):
    import torch
    return torch.from_numpy(mat.data.view(np.int16)).view(torch.bfloat16).pin_memory()


def run_workload(args, rank, world, local):
    """One timed step of a --workload other than the single layer: the
    split / quantize phase, then the products, captured as one CUDA graph
    and replayed with L2 flushed before every step."""
    import torch
    from spectral_domain_quantization_b200 import api

    assert torch.cuda.is_available(), "bench needs a GPU"
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if not api.lib().metis_device_supported():
        raise RuntimeError("metis needs an sm_100 (B200) device")
    wl = WORKLOADS[args.workload](dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def step():
        wl.split()
        wl.products()

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

    g_step = capture(step)
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

    g_split = capture(wl.split)
    ms_split = time_graph(g_split, args.steps, 3)
    wl.split()
    g_prod = capture(wl.products)
    ms_prod = time_graph(g_prod, args.steps, 3)
    plain_flops, plain_name = wl.plain()
    g_plain = capture(wl.plain)
    ms_plain = time_graph(g_plain, args.steps, 3)

    e2e = None
    if not args.no_e2e:
        # every step uploads its inputs from pinned host memory and copies its
        # outputs back, on the compute stream, inside the timed region
        outs = wl.outputs()
        out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]

        def e2e_step():
            for k, h in wl.host.items():
                wl.dev[k].copy_(h, non_blocking=True)
            g_step.replay()
            for h, o in zip(out_host, outs):
                h.copy_(o, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, world)
        e2e = {"value": world * wl.flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(sum(h.numel() * h.element_size() for h in wl.host.values())),
               "d2h_bytes_per_step": int(sum(o.numel() * o.element_size() for o in outs)),
               "pipelining": "none: uploads, the step and the downloads in order on one stream"}

    hbm, bf16_tf, peak_kind = measured_peaks()
    fp4_peak = 4.0 * bf16_tf
    achieved = plain_flops / (ms_plain * 1e-3) / 1e12
    value = world * wl.flops / (ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        t, _, desc = wl.oracle_sample()
        cpu = {"value": wl.flops / t / 1e12, "unit": "TFLOPS", "cores": blas_threads(), "kind": "oracle",
               "sample": desc, "full_step_ms_extrapolated": t * 1e3}
    if rank == 0:
        split_gbs = wl.split_bytes / (ms_split * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp4 (e2m1 with nvfp4 / mxfp4 scales; fp32 accumulate)", "data": "synthetic",
            "config": dict(wl.config, l2="flushed (512 MB write) before every timed step"),
            "frac_of_fp4_peak": value / world / fp4_peak,
            "split_quantize_us_per_layer": ms_split * 1e3,
            "breakdown_us": {"split_quantize": ms_split * 1e3, "products": ms_prod * 1e3,
                             "fp4_gemm_kernel": ms_plain * 1e3},
            "hbm": {"split_quantize": {"algorithmic_bytes": wl.split_bytes, "achieved_gbs": split_gbs,
                                       "peak_gbs": hbm, "frac": split_gbs / hbm, "peak_source": peak_kind}},
            "roofline": {"kernel": plain_name, "bound": "tensor", "achieved": achieved, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                         "peak_source": f"{peak_kind} bf16 {bf16_tf} TFLOP/s x 4 (nominal FP4/bf16 ratio)",
                         "traffic": None},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    del g_step, g_split, g_prod, g_plain


def run_profile(args, local):
    """The step, eagerly and untimed: a short launch list for profilers
    (the single-layer step, or the --workload step)."""
    import torch
    from spectral_domain_quantization_b200 import api, inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.workload != "layer_4096":
        wl = WORKLOADS[args.workload](dev)
        for _ in range(args.profile_steps):
            wl.split()
            wl.products()
        torch.cuda.synchronize()
        print(json.dumps({"profile_steps": args.profile_steps, "workload": args.workload}), flush=True)
        return
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
        # the plain-operand product whose kernel the roofline times (the
        # third gemm_fp4_kernel launch of a step)
        api.linear_fwd(api.Operand(xq), api.Operand(s.R_cols), M, N, K, Y=Y, dev_status=status)
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
        elif args.workload != "layer_4096":
            run_workload(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
