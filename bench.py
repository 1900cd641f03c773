#!/usr/bin/env python
"""Benchmark of the B200 RT-Lynx online 2:4 activation-sparse linear layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle, timed as it stands

One step = one ``lynx_linear`` call (sparsify + LoRA-down pass, sparse GEMM with
LoRA-up and bias epilogue) on one batch of the workload, inputs resident in
HBM.  L2 is flushed (256 MiB write) before every step, outside the timed step;
each step is timed with CUDA events on the launching stream.  The metric is the
dense-equivalent throughput 2*M*N*K / t.  Alongside: a dense bf16 GEMM of the
same shape (torch.matmul / cuBLAS, comparison only), this library's dense path,
the per-kernel split (sparsify pass vs GEMM), an end-to-end number through the
same call with pinned host buffers, clocks sampled during the timed region,
the roofline of the dominant kernel and the CPU oracle's throughput on a
bounded sample.

Multi-GPU (torchrun, one process per GPU): token rows are independent, so each
rank runs its own batch of the workload (weak scaling, no data-path
collective); the step time is the maximum over ranks.
"""
import argparse
import datetime
import json
import math
import os
import platform
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-act linear dense-equiv TFLOP/s (2MNK/t) & speedup vs dense bf16 GEMM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per launch of the sparse GEMM kernel from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum), with the hash of the
# GEMM's sources at the capture: the bench reports the figure only while the
# sources still hash the same, else null ("stale").
# The sources each kernel's launch depends on (the host code sets its grid and raster).
KERNEL_SOURCES = {
    "gemm": ("gemm_pair_kernel.cu", "lynx_ptx.cuh", "lynx_internal.h", "lynx_act.cuh", "lynx_select.cuh",
             "lynx_api.cu"),
    "sparsify": ("sparsify_kernel.cu", "lynx_select.cuh", "lynx_ptx.cuh", "lynx_internal.h", "lynx_api.cu"),
}
# dram__bytes_read.sum + dram__bytes_write.sum per launch from one ncu capture per
# workload (profile_layer, L2 flushed before the call), stamped with the hash of
# the kernel's sources at capture; reported only while the sources still hash so.
DRAM_TRAFFIC = {
    "gemm": {"src": "581e8f60d635", "captured": "2026-12-03",
             "bytes": {"mlp_up": 185362944, "attn_out": 44645888, "mlp_down": 311768320}},
    "sparsify": {"src": "d5bc16ab1aa1", "captured": "2026-12-03",
                 "bytes": {"mlp_up": 28757504, "attn_out": 25598976, "mlp_down": 149431296}},
}

def uses_pair_gemm(M, N, K):
    """The library's choice: the CTA-pair GEMM unless the shape cannot feed it."""
    return M > 128 and N >= 256 and K % 128 == 0


def launches_per_linear(M, N, K, skip=False, lora=True):
    """Kernels one lynx_linear call launches: the sparsify pass (or, on the dense
    path, the LoRA-down pass), a finalize kernel unless the pair GEMM combines
    the pass's partials itself, and the GEMM."""
    if skip and not lora:
        return 1
    return 2 if uses_pair_gemm(M, N, K) else 3


def gemm_kernel_name(M, N, K):
    """Name of the GEMM kernel the library picks for a sparse call of this shape."""
    if uses_pair_gemm(M, N, K):
        return "lynx_gemm_pair_kernel<1> (CTA pair, 256x256 tiles)"
    return f"lynx_gemm_kernel<{256 if N >= 1024 else 128},1>"


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["lynx", "reference"], default="lynx")
    ap.add_argument("--workload", default="mlp_up")
    ap.add_argument("--act", choices=["none", "gelu_tanh"], default="none",
                    help="activation applied in the GEMM epilogue (lynx_linear_act); the "
                         "comparisons then apply the same activation as a separate pass")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="approximate CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per_config block (the other DiT shapes)")
    ap.add_argument("--gather-y", action="store_true",
                    help="with --gpus N > 1: also time the layer followed by an all-gather of Y "
                         "(every rank ends with all N x M rows), reported as y_gather")
    ap.add_argument("--sweep-schedule", choices=["serial", "overlap", "overlap_chunks2"], default="serial",
                    help="--workload sweep: the schedule the headline times (all three are reported)")
    ap.add_argument("--only-linear", action="store_true",
                    help="time the layer only (no comparisons, e2e or CPU baseline); "
                         "the short launch sequence used for ncu captures")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value, world):
    """Max of a float over all ranks (a timing reduction, not part of the layer)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank, ms_max, world):
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; no setting is changed)

class ClockSampler:
    REASONS = {
        0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
    }

    def __init__(self, torch_device_index):
        self.samples = []
        self.reasons = 0
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            import torch

            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hh)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hh
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.h = h
            self.nv = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are informative only
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                r = get_reasons(self.h)
                self.samples.append((float(mhz), int(util), int(r)))
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(0.01)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable: " + getattr(self, "err", "")}
        busy = [s for s in self.samples if s[1] > 0] or self.samples
        reasons = 0
        for s in busy:
            reasons |= s[2]
        names = sorted(n for bit, n in self.REASONS.items() if reasons & bit)
        return {"sm_mhz": statistics.median(s[0] for s in busy) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(busy)}


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample of the workload

def oracle_sample(inp, rows, skip=False, act="none"):
    import oracle

    X = inp["X"][:rows]
    t0 = time.perf_counter()
    Y, _, _ = oracle.linear(X, inp["W"], inp["bias"], inp["A"], inp["B"], skip=skip)
    if act == "gelu_tanh":
        oracle.gelu_tanh(Y)
    return time.perf_counter() - t0


def calibrate_oracle_rows(inp, target_s, M):
    import oracle

    cores = oracle.num_threads()
    rows = max(1, cores)
    t = oracle_sample(inp, rows)
    while t < target_s / 4 and rows < M:
        rows = min(M, int(rows * max(2.0, target_s / max(t, 1e-3) / 2)))
        t = oracle_sample(inp, rows)
    rows = min(M, max(1, int(rows * target_s / max(t, 1e-3))))
    return rows, cores


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def single_thread_sample(inp, shape, target_s):
    """The same oracle on one thread, on whole rows for about `target_s`."""
    import oracle

    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        rows = 1
        t = oracle_sample(inp, rows)
        rows = min(shape.M, max(1, int(rows * target_s / max(t, 1e-3))))
        t = oracle_sample(inp, rows)
    finally:
        oracle.set_num_threads(cores)
    return {"value": 2.0 * rows * shape.N * shape.K / t / 1e12, "unit": "TFLOP/s", "cores": 1,
            "sample": f"{rows} token rows, {t:.1f} s"}


def cpu_baseline(inp, shape, target_s, act="none"):
    rows, cores = calibrate_oracle_rows(inp, target_s, shape.M)
    t = oracle_sample(inp, rows, act=act)
    flops = 2.0 * rows * shape.N * shape.K
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} of {shape.M} token rows of {shape.name} (rows are independent), "
                      f"full N={shape.N} and K={shape.K}, fp64 C oracle, {t:.1f} s",
            "cpu": cpu_model(),
            "single_thread": single_thread_sample(inp, shape, min(3.0, target_s / 4))}


# ---------------------------------------------------------------------------


def workload_desc(shape):
    kind = "GELU(tanh) inputs" if shape.x_kind == "gelu" else "8% N(0,1) / 92% N(0,0.05) mixture"
    return (f"{shape.name}: X[{shape.M},{shape.K}] -> Y[{shape.M},{shape.N}], LoRA r={shape.r}, "
            f"bias, {kind}")


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from activation_sparse_gemm_lynx_b200 import workloads
    import oracle

    shape = workloads.CONFIGS[args.workload]
    inp = workloads.make_config_inputs(args.workload)
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    rows, cores = calibrate_oracle_rows(inp, per_step, shape.M)
    for _ in range(args.warmup):
        oracle_sample(inp, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(inp, rows)
    t = (time.perf_counter() - t0) / max(1, args.steps)
    value = 2.0 * rows * shape.N * shape.K / t / 1e12
    sample = (f"each step: {rows} of {shape.M} token rows of {shape.name} (rows are independent), "
              f"full N and K, fp64 C oracle on {cores} threads")
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": workload_desc(shape), "M": shape.M, "N": shape.N, "K": shape.K,
                   "r": shape.r, "rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out), flush=True)
    return 0


class LayerTimer:
    """Device-resident inputs of one workload and the timing loops over them
    (CUDA events on the launching stream, L2 flushed before every step)."""

    def __init__(self, name, rank, act_name, flush):
        import numpy as np
        import torch

        from activation_sparse_gemm_lynx_b200 import lynx, workloads

        self.lynx, self.torch = lynx, torch
        self.workload, self.act_name = name, act_name
        self.shape = workloads.CONFIGS[name]
        M, N, K, r = self.shape.M, self.shape.N, self.shape.K, self.shape.r
        self.inp = workloads.make_rank_inputs(name, rank)

        def dev(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

        self.X, self.W, self.bias, self.A, self.B = (dev(self.inp[k]) for k in ("X", "W", "bias", "A", "B"))
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        self.Yd = torch.empty_like(self.Y)
        self.ws = torch.empty(lynx.lynx_workspace_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
        self.flush = flush
        self.act = {"none": lynx.LYNX_ACT_NONE, "gelu_tanh": lynx.LYNX_ACT_GELU_TANH}[act_name]

    def step_linear(self, skip=False):
        if self.act == self.lynx.LYNX_ACT_NONE and not skip:
            self.lynx.lynx_linear(self.X, self.W, self.bias, self.A, self.B, Y=self.Y, workspace=self.ws)
        else:
            self.lynx.lynx_linear_act(self.X, self.W, self.bias, self.A, self.B, skip_sparsify=skip,
                                      act=self.act, Y=self.Y, workspace=self.ws)

    def step_dense_torch(self):
        self.torch.matmul(self.X, self.W.t(), out=self.Yd)
        if self.act != self.lynx.LYNX_ACT_NONE:
            self.torch.nn.functional.gelu(self.Yd, approximate="tanh")

    def step_fused(self):
        self.lynx.lynx_linear_fused(self.X, self.W, self.bias, self.A, self.B, Y=self.Y, workspace=self.ws)

    def step_unfused_act(self):
        # the plain layer, then the activation as a pass of its own over Y
        self.lynx.lynx_linear(self.X, self.W, self.bias, self.A, self.B, Y=self.Y, workspace=self.ws)
        self.torch.nn.functional.gelu(self.Y, approximate="tanh")

    def timed(self, step, n, split=False, part=0):
        """Per-step device times (ms) of n steps, L2 flushed before each.  With
        split, also the times up to and after the library's split event; with
        part 1 / 2, lynx_linear runs only its first kernel / the rest."""
        torch, lynx = self.torch, self.lynx
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
        for trio in ev:        # create the CUDA events up front
            for e in trio:
                e.record()
        torch.cuda.synchronize()
        lynx.lynx_profile_set_part(part)
        try:
            for i in range(n):
                self.flush.zero_()
                if split:
                    lynx.lynx_profile_set_split_event(ev[i][1])
                ev[i][0].record()
                step()
                ev[i][2].record()
        finally:
            lynx.lynx_profile_set_split_event(None)
            lynx.lynx_profile_set_part(0)
        torch.cuda.synchronize()
        tot = [ev[i][0].elapsed_time(ev[i][2]) for i in range(n)]
        if split:
            first = [ev[i][0].elapsed_time(ev[i][1]) for i in range(n)]
            second = [ev[i][1].elapsed_time(ev[i][2]) for i in range(n)]
            return tot, first, second
        return tot

    def sparsify_back_to_back(self, reps=12):
        """Average device time (ms) of one sparsify pass (lynx_linear's first
        kernel alone) launched back to back over distinct copies of X whose
        total exceeds the 126 MB L2 by half again, so that every launch reads
        its X from DRAM with no flush between launches (each launch follows the
        previous one as in a layer: programmatic launch, then its wait)."""
        torch, lynx = self.torch, self.lynx
        xbytes = self.X.numel() * self.X.element_size()
        copies = [self.X.clone() for _ in range(max(2, -(-(192 << 20) // xbytes)))]
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        lynx.lynx_profile_set_part(1)
        try:
            for x in copies + copies:
                lynx.lynx_linear(x, self.W, self.bias, self.A, self.B, Y=self.Y, workspace=self.ws)
            self.flush.zero_()
            ev[0].record()
            for i in range(reps):
                for x in copies:
                    lynx.lynx_linear(x, self.W, self.bias, self.A, self.B, Y=self.Y, workspace=self.ws)
                ev[i + 1].record()
        finally:
            lynx.lynx_profile_set_part(0)
        torch.cuda.synchronize()
        # the median over the rounds of one launch per copy (a slow round is not averaged in)
        per_round = [ev[i].elapsed_time(ev[i + 1]) / len(copies) for i in range(reps)]
        del copies
        return statistics.median(per_round)

    def parts(self, n):
        """Time of the layer's parts, each run alone (means over n steps):
        the sparsify / LoRA-down kernel (events around that one launch, and
        back to back over copies of X larger than L2), the GEMM (from an event
        recorded after the reset of its state words to the end), and the two
        kernels of a call split by an event between them."""
        mean = statistics.mean
        sp_alone = mean(self.timed(self.step_linear, n, part=1))
        sp_b2b = self.sparsify_back_to_back()
        _, _, gemm_alone = self.timed(self.step_linear, n, split=True, part=2)
        split_tot, split_sp, split_gemm = self.timed(self.step_linear, n, split=True)
        return {"sparsify_kernel": sp_alone, "sparsify_back_to_back": sp_b2b, "gemm_kernel": mean(gemm_alone),
                "linear_split": mean(split_tot), "split_first": mean(split_sp),
                "split_second": mean(split_gemm)}


def src_hash(files):
    """Short hash of the named CUDA sources (the build a stored ncu figure belongs to)."""
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "activation_sparse_gemm_lynx_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def stored_traffic(kernel, workload):
    """ncu's DRAM bytes per launch of `kernel` ("gemm" or "sparsify") on this
    workload, if the stored capture was taken on the kernel's sources as they
    stand; else (None, why)."""
    rec = DRAM_TRAFFIC[kernel]
    if workload not in rec["bytes"]:
        return None, "not captured for this workload"
    now = src_hash(KERNEL_SOURCES[kernel])
    if rec["src"] != now:
        return None, f"stale: captured on sources {rec['src']}, kernel now {now}"
    return rec["bytes"][workload], f"ncu capture of {rec['captured']} (sources {rec['src']})"


def layer_summary(lt, ms_linear, parts, dense_ms, peaks, clock_info=None, fused_ms=None):
    M, N, K, r = lt.shape.M, lt.shape.N, lt.shape.K, lt.shape.r
    flops = 2.0 * M * N * K
    sparse_peak = 2.0 * peaks["bf16_tflops"]
    gemm_tflops = flops / (parts["gemm_kernel"] * 1e-3) / 1e12
    sp_bytes = 2 * M * K + M * K + lt.lynx.lynx_meta_bytes(M, K) + 2 * M * r + 4 * M + 2 * r * K
    out = {
        "value": flops / (ms_linear * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms_linear,
        "M": M, "N": N, "K": K, "r": r,
        "speedup_vs_dense_bf16": dense_ms / ms_linear,
        "sparsify_overhead": max(0.0, 1.0 - parts["gemm_kernel"] / ms_linear),
        "gemm_frac": gemm_tflops / sparse_peak,
        "gemm_tflops": gemm_tflops,
        "gemm_traffic": stored_traffic("gemm", lt.workload)[0] if lt.act_name == "none" else None,
        "sparsify_traffic": stored_traffic("sparsify", lt.workload)[0],
        "sparsify_frac": sp_bytes / (parts["sparsify_back_to_back"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "ms": {"sparsify_kernel": parts["sparsify_kernel"], "sparsify_back_to_back": parts["sparsify_back_to_back"],
               "gemm_kernel": parts["gemm_kernel"],
               "dense_torch_matmul": dense_ms},
    }
    if fused_ms is not None:
        # the fully fused variant (selection inside the GEMM), for comparison
        out["fused_variant"] = {"ms_per_step": fused_ms, "value": flops / (fused_ms * 1e-3) / 1e12,
                                "vs_two_pass": ms_linear / fused_ms}
    if clock_info is not None:
        out["clocks"] = clock_info
    return out


def run_lynx(args):
    import torch

    from activation_sparse_gemm_lynx_b200 import lynx

    rank, local_rank, world = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    lynx.library()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device="cuda")
    lt = LayerTimer(args.workload, rank, args.act, flush)
    shape = lt.shape
    M, N, K, r = shape.M, shape.N, shape.K, shape.r
    Xh = torch.from_numpy(lt.inp["X"].view("int16")).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    act = lt.act

    ws_host = torch.empty(lynx.lynx_linear_host_workspace_bytes(M, N, K, r), dtype=torch.uint8,
                          device="cuda")

    def step_e2e():
        # the C-ABI call on host buffers: copies in, the layer and copies out,
        # pipelined over row chunks inside the library
        if act == lynx.LYNX_ACT_NONE:
            lynx.lynx_linear_host(Xh, lt.W, lt.bias, lt.A, lt.B, Y_host=Yh, workspace=ws_host)
        else:
            lynx.lynx_linear_host_act(Xh, lt.W, lt.bias, lt.A, lt.B, act=act, Y_host=Yh,
                                      workspace=ws_host)

    # warm-up (untimed)
    for _ in range(args.warmup):
        lt.step_linear()
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    if st != lynx.LYNX_OK:
        raise RuntimeError(f"device status after warm-up: {st} code {code:#x}")

    # the parts of the layer, each in a loop of its own before the timed steps
    # (an event between the kernels keeps the GEMM's launch from overlapping the
    # pass's tail, so the headline loop runs without it)
    ncmp = max(3, min(args.steps, 50))
    parts = lt.parts(ncmp)

    clocks = ClockSampler(local_rank)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    tot = lt.timed(lt.step_linear, args.steps)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    barrier(world)
    st, code = lynx.lynx_check_error()
    if st != lynx.LYNX_OK:
        raise RuntimeError(f"device status after timing: {st} code {code:#x}")
    total_ms = max_over_ranks(sum(tot), world)
    ms_step = total_ms / args.steps

    if args.only_linear:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "ms_per_step": ms_step,
                              "sparsify_ms": parts["sparsify_kernel"], "gemm_ms": parts["gemm_kernel"],
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "only_linear": True}), flush=True)
        return 0

    # comparisons (same process, same loop structure)
    for _ in range(3):
        lt.step_dense_torch()
    dense_ms = max_over_ranks(statistics.mean(lt.timed(lt.step_dense_torch, ncmp)), world)
    for _ in range(3):
        lt.step_linear(skip=True)
    lynx_dense_ms = max_over_ranks(statistics.mean(lt.timed(lambda: lt.step_linear(skip=True), ncmp)),
                                   world)
    for _ in range(3):
        step_e2e()
    e2e_ms = max_over_ranks(statistics.mean(lt.timed(step_e2e, ncmp)), world)
    unfused_ms = None
    if act != lynx.LYNX_ACT_NONE:
        for _ in range(3):
            lt.step_unfused_act()
        unfused_ms = max_over_ranks(statistics.mean(lt.timed(lt.step_unfused_act, ncmp)), world)
    parts = {k: max_over_ranks(v, world) for k, v in parts.items()}

    flops = 2.0 * M * N * K
    peaks = load_peaks()
    sparse_peak = 2.0 * peaks["bf16_tflops"]
    gemm_tflops = flops / (parts["gemm_kernel"] * 1e-3) / 1e12
    sp_bytes = 2 * M * K + M * K + lynx.lynx_meta_bytes(M, K) + 2 * M * r + 4 * M + 2 * r * K
    sp_gbs = sp_bytes / (parts["sparsify_back_to_back"] * 1e-3) / 1e9
    traffic, traffic_note = stored_traffic("gemm", args.workload) if act == lynx.LYNX_ACT_NONE \
        else (None, "not captured with the epilogue activation")
    sp_traffic, sp_traffic_note = stored_traffic("sparsify", args.workload)

    result = {
        "metric": METRIC,
        "value": aggregate_tflops(flops, ms_step, world),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded numpy draws rounded to bf16; random weights)",
        "config": {
            "workload": workload_desc(shape) + ("" if act == lynx.LYNX_ACT_NONE
                                                else ", GELU(tanh) applied in the GEMM epilogue"),
            "M": M, "N": N, "K": K, "r": r,
            "l2": "flushed before every step (256 MiB write, outside the timed step)",
            "parallelism": f"dp{world} (independent token-row batches per GPU, no collective)",
        },
        "speedup_vs_dense_bf16": dense_ms / ms_step,
        "sparsify_overhead": max(0.0, 1.0 - parts["gemm_kernel"] / ms_step),
        "overhead_note": "1 - t(GEMM kernel alone) / t(layer): the time the layer adds to its GEMM",
        "breakdown_ms": {"linear": ms_step, "sparsify_kernel": parts["sparsify_kernel"],
                         "sparsify_back_to_back": parts["sparsify_back_to_back"],
                         "gemm_kernel": parts["gemm_kernel"], "linear_split": parts["linear_split"],
                         "split_sparsify_pass": parts["split_first"], "split_gemm": parts["split_second"],
                         "dense_torch_matmul": dense_ms, "lynx_dense_path": lynx_dense_ms},
        "roofline": {
            "bound": "tensor", "kernel": gemm_kernel_name(M, N, K),
            "achieved": gemm_tflops, "peak": sparse_peak, "unit": "TFLOP/s",
            "frac": gemm_tflops / sparse_peak, "traffic": traffic, "traffic_note": traffic_note,
            "peak_note": f"2 x {peaks['source']} dense bf16 burst ({peaks['bf16_tflops']} TFLOP/s); "
                         "2:4 sparse runs at twice the dense rate",
            "work": "2*M*N*K dense-equivalent flops per launch; time: the GEMM launched alone",
        },
        "roofline_sparsify": {
            "bound": "hbm", "kernel": "sparsify_kernel", "achieved": sp_gbs,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": sp_gbs / peaks["hbm_gbs"],
            "traffic": sp_traffic, "traffic_note": sp_traffic_note,
            "work": "algorithmic bytes X read 2MK + vals MK + meta MK/8 + T 2Mr + s 4M + A 2rK; "
                    "time: the kernel launched back to back over copies of X larger than L2 (average per launch; "
                    "breakdown_ms.sparsify_kernel is one launch after an L2 flush, dispatch gap included)",
            "time_ms": parts["sparsify_back_to_back"],
        },
        "e2e": {"value": aggregate_tflops(flops, e2e_ms, world), "unit": "TFLOP/s",
                "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 2 * M * N,
                "ms_per_step": e2e_ms,
                "note": "lynx_linear_host on pinned host X and Y: the copies in, the layer and the "
                        "copies out inside each step, overlapped over row chunks; weights resident"},
        "gpu_launches": launches_per_linear(M, N, K) * args.steps,
        "clocks": clock_info,
    }

    if unfused_ms is not None:
        result["config"]["act"] = args.act
        result["speedup_vs_unfused_act"] = unfused_ms / ms_step
        result["breakdown_ms"]["linear_then_separate_act"] = unfused_ms
        result["dense_note"] = "torch.matmul then torch GELU (tanh) as a separate pass"

    if args.gather_y and world > 1:
        # the row-sharded layer followed by an NCCL all-gather of Y's row blocks
        from activation_sparse_gemm_lynx_b200 import sharded

        def step_gather():
            lt.step_linear()
            sharded.gather_rows(lt.Y, world * M)

        for _ in range(3):
            step_gather()
        g_ms = max_over_ranks(statistics.mean(lt.timed(step_gather, ncmp)), world)
        result["y_gather"] = {"ms_per_step": g_ms, "value": aggregate_tflops(flops, g_ms, world),
                              "unit": "TFLOP/s", "gathered_bytes_per_rank": 2 * M * N * (world - 1),
                              "note": "lynx_linear on each rank's rows, then all_gather_into_tensor of Y"}

    # the other DiT shapes of the same targets, measured in this run the same
    # way (fewer steps); the headline stays the selected workload
    if not args.no_per_config and act == lynx.LYNX_ACT_NONE:
        per = {}
        def fused_time(t):
            for _ in range(3):
                t.step_fused()
            return max_over_ranks(statistics.mean(t.timed(t.step_fused, ncmp)), world)

        for name in ("attn_out", "mlp_up", "mlp_down"):
            if name == args.workload:
                per[name] = layer_summary(lt, ms_step, parts, dense_ms, peaks, clock_info, fused_time(lt))
                continue
            other = LayerTimer(name, rank, "none", flush)
            for _ in range(max(3, args.warmup)):
                other.step_linear()
            torch.cuda.synchronize()
            o_parts = {k: max_over_ranks(v, world) for k, v in other.parts(ncmp).items()}
            ck = ClockSampler(local_rank)
            barrier(world)
            torch.cuda.synchronize()
            ck.start()
            o_ms = max_over_ranks(statistics.mean(other.timed(other.step_linear, ncmp)), world)
            o_clock = ck.stop()
            for _ in range(3):
                other.step_dense_torch()
            o_dense = max_over_ranks(statistics.mean(other.timed(other.step_dense_torch, ncmp)), world)
            per[name] = layer_summary(other, o_ms, o_parts, o_dense, peaks, o_clock, fused_time(other))
            per[name]["steps"] = ncmp
            del other
        st, code = lynx.lynx_check_error()
        if st != lynx.LYNX_OK:
            raise RuntimeError(f"device status after the per-config runs: {st} code {code:#x}")
        result["per_config"] = per

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(lt.inp, shape, args.cpu_seconds, act=args.act)

    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def run_sweep(args):
    """The DiT block sweep: 8 blocks x {qkv, out, up, down} linears at M = 8192,
    2 blocks left dense (skip_sparsify), fresh seeded inputs per linear, all 32
    calls captured once in a CUDA graph and replayed as one step."""
    import torch

    from activation_sparse_gemm_lynx_b200 import lynx, workloads
    from activation_sparse_gemm_lynx_b200.sweep import LinearSweep

    rank, local_rank, world = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    lynx.library()
    plan = workloads.sweep_plan()
    layers = []
    gelu_up = args.act == "gelu_tanh"
    for (_b, name, M, K, N, kind, skip, seed) in plan:
        inp = workloads.make_linear_inputs(M, K, N, seed=seed, x_kind=kind)
        inp["skip"] = skip
        if gelu_up and name == "up":
            inp["act"] = lynx.LYNX_ACT_GELU_TANH
        layers.append(inp)
    sweep = LinearSweep(layers)
    del layers
    flops = sweep.dense_flops
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device="cuda")

    def timed(step, n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for a, b in ev:
            a.record()
            b.record()
        torch.cuda.synchronize()
        for i in range(n):
            flush.zero_()
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    sweep.run()  # one-time set-up of the library happens outside the capture
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    if st != lynx.LYNX_OK:
        raise RuntimeError(f"device status after the first pass: {st} code {code:#x}")
    eager_before = timed(sweep.run, 5)
    # the other schedules, each run once eagerly before its capture
    schedules = {"serial": (False, 1), "overlap": (True, 1), "overlap_chunks2": (True, 2)}
    graphs = {}
    for name, (overlapped, chunks) in schedules.items():
        if overlapped:
            sweep.run_overlapped(chunks)
            torch.cuda.synchronize()
        graphs[name] = sweep.capture(overlapped, chunks)
    sweep.graph = graphs[args.sweep_schedule]
    for _ in range(args.warmup):
        sweep.replay()
    clocks = ClockSampler(local_rank)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    tot = timed(sweep.replay, args.steps)
    clock_info = clocks.stop()
    barrier(world)
    st, code = lynx.lynx_check_error()
    if st != lynx.LYNX_OK:
        raise RuntimeError(f"device status after timing: {st} code {code:#x}")
    ms_step = max_over_ranks(sum(tot), world) / args.steps
    schedule_ms = {}
    for name, g in graphs.items():
        for _ in range(3):
            g.replay()
        schedule_ms[name] = max_over_ranks(statistics.mean(timed(g.replay, max(3, min(args.steps, 20)))),
                                           world)
    st, code = lynx.lynx_check_error()
    for side in sweep.side_streams():
        if st == lynx.LYNX_OK:
            st, code = lynx.lynx_check_error(side)
    if st != lynx.LYNX_OK:
        raise RuntimeError(f"device status after the schedules: {st} code {code:#x}")
    # eager launches (host work in every step) before and after the graph loop
    eager_ms = max_over_ranks(statistics.mean(eager_before + timed(sweep.run, 5)), world)

    # the same 32 products as plain dense bf16 GEMMs (cuBLAS), also one graph
    outs = [torch.empty_like(t["Y"]) for t in sweep.layers]

    def dense_all():
        for t, y in zip(sweep.layers, outs):
            torch.matmul(t["X"], t["W"].t(), out=y)
            if t["act"] != lynx.LYNX_ACT_NONE:
                torch.nn.functional.gelu(y, approximate="tanh")

    dense_all()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        dense_all()
    for _ in range(3):
        g.replay()
    dense_ms = max_over_ranks(statistics.mean(timed(g.replay, max(3, min(args.steps, 20)))), world)
    del g
    skipped = sorted({b for (b, *_rest) in plan if _rest[5]})
    result = {
        "metric": METRIC,
        "value": aggregate_tflops(flops, ms_step, world),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded numpy draws rounded to bf16; random weights)",
        "config": {
            "workload": "sweep: 8 DiT blocks x {qkv 3072->9216, out 3072->3072, up 3072->12288, "
                        "down 12288->3072 (GELU inputs)} at M=8192, LoRA r=64, bias; "
                        f"blocks {skipped} dense (skip_sparsify)",
            "M": workloads.SWEEP_M, "layers": len(plan),
            "l2": "flushed before every step (256 MiB write, outside the timed step)",
            "parallelism": f"dp{world} (independent token-row batches per GPU, no collective)",
            "graph": "the 32 lynx_linear calls replayed from one CUDA graph",
            "schedule": {"serial": "the calls in order on one stream",
                         "overlap": "each layer's sparsify pass on a side stream, its GEMM on the main "
                                    "stream, two workspaces in turn",
                         "overlap_chunks2": "as overlap, each layer in two row blocks"}[args.sweep_schedule],
            **({"act": "GELU(tanh) on the 8 MLP up-projection outputs: in the GEMM epilogue here, "
                       "as a separate torch pass after each matmul in the cuBLAS graph"}
               if gelu_up else {}),
        },
        "speedup_vs_dense_bf16": dense_ms / ms_step,
        "breakdown_ms": {"sweep_graph": ms_step, "sweep_eager": eager_ms,
                         "dense_torch_matmul_graph": dense_ms,
                         **{f"sweep_graph_{k}": v for k, v in schedule_ms.items()}},
        "gpu_launches": args.steps * sum(
            launches_per_linear(r1 - r0, t["shape"][2], t["shape"][1], skip=t["skip"], lora=t["A"] is not None)
            for (t, r0, r1) in sweep.work_items(schedules[args.sweep_schedule][1])),
        "clocks": clock_info,
    }
    if world > 1:
        import torch.distributed as dist

        sweep.graph = None
        graphs.clear()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "sweep":
        return run_sweep(args)
    return run_lynx(args)


if __name__ == "__main__":
    sys.exit(main())
