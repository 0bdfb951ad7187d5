#!/usr/bin/env python
"""Benchmark of the B200 SmoothQuant W8A8 INT8 linear layer.

One step = one pass of the layer's hot path over one batch: per-token
dynamic INT8 quantisation of X with the SmoothQuant 1/s fold, then the
INT8 x INT8 GEMM with the fused per-token x per-channel BF16 epilogue, on the
prefill workload M=8192 tokens, K=5120, N=34816 (fused gate/up shape).
The printed metric is TOPS (2*M*N*K per step, quantisation included in the
time), over a short burst of steps (`value`) and over two seconds of steps
(`sustained`, under the power cap), with the device's INT8 tensor rate
measured by the library's issue-rate probe for each.  The same run also
measures the decode W8A8 shape, the gs128 variant, the W8A16 (down_proj)
variant at M = 1, 16, 8192, and the next rows: fused RMSNorm quantisation,
per-group INT8 / FP8 activation quantisation, per-group x gs128 and FP8
block GEMMs, and group-wise W8A16.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

N > 1 (under torchrun) runs N independent replicas of the same workload,
one per GPU (the layer has no exchange step on one GPU); value is the sum
of the work over the max of the per-rank device times.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "W8A8 GEMM TOPS incl. per-token quant (% of INT8 peak); W8A16 GB/s at M≤16"
INT8_PER_BF16 = 2.0          # dense INT8 ops per dense BF16 flop (4.5 / 2.25 PFLOP/s nominal)
INT8_NOMINAL_TOPS = 4500.0   # dense INT8, nominal B200


def gemm_traffic():
    """DRAM bytes per launch of the prefill GEMM from the committed ncu record,
    or None if the kernel sources changed since it was captured."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "gemm2_w8a8_prefill_traffic.json")))
        h = hashlib.sha256()
        for src in rec["sources"]:
            h.update(open(os.path.join(ROOT, src), "rb").read())
        return rec["traffic_bytes_per_launch"] if h.hexdigest() == rec["sources_sha256"] else None
    except Exception:
        return None


def load_peaks():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------- clock sampler
class ClockSampler(threading.Thread):
    """Samples the SM clock and clock-event reasons through NVML every 5 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device: int):
        super().__init__(daemon=True)
        self.samples = []
        self.reasons = 0
        self.stop_evt = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = self._handle(device)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception:
            self.ok = False

    def _handle(self, device):
        nv = self.nv
        try:
            p = torch.cuda.get_device_properties(device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(0)

    def run(self):
        if not self.ok:
            return
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(self.get_reasons(self.h))
            except Exception:
                pass
            time.sleep(0.005)

    def result(self):
        self.stop_evt.set()
        self.join(timeout=2)
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        busy = [s for s in self.samples if s > 0]
        bins = {}
        for v in busy:
            b = int(v // 100 * 100)
            bins[b] = bins.get(b, 0) + 1
        return {"sm_mhz": statistics.median(busy or self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1],
                "samples": len(self.samples),
                "mhz_bins": {str(k): bins[k] for k in sorted(bins)}}


# -------------------------------------------------------------------- helpers
def algo_bytes_quant(M, K):
    return 2 * M * K + 4 * K + M * K + 4 * M


def algo_bytes_w8a8(M, N, K, gs=False):
    scales = 4 * N * (K // 128) if gs else 4 * N
    return M * K + N * K + 4 * M + scales + 2 * M * N


def algo_bytes_w8a16(M, N, K):
    return 2 * M * K + N * K + 4 * N + 2 * M * N


def time_batches(fn, iters, warmup=3):
    """Device time per call of fn (back-to-back launches on the current stream)."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(iters):
        fn(i)
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters * 1e-3


def time_graph(fn, calls, reps=5):
    """Device time per call of fn, with `calls` calls captured in one CUDA graph
    (so host launch overhead is not measured) and the graph replayed `reps`
    times back to back."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):           # eager warm-up on the capture stream:
        for i in range(3):               # creates its workspace, sets attributes
            fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(calls):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / (reps * calls) * 1e-3


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def replica_collectives(world: int, dev: torch.device):
    """The only collectives of the replicas: a barrier (plus a device
    synchronize on CUDA) and the maximum of a per-rank time.  Any backend:
    NCCL on the GPUs, gloo in the CPU tests."""
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()
        if dev.type == "cuda":
            torch.cuda.synchronize(dev)

    def max_over_ranks(v: float) -> float:
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def whole_job_tops(ops_per_step: float, steps: int, world: int, seconds: float) -> float:
    """Every replica runs `steps` steps; the job's rate is all ranks' work
    over the slowest rank's time."""
    return ops_per_step * steps * world / seconds / 1e12


# ------------------------------------------------------------ CPU oracle leg
def oracle_sample(wl, target_s: float, max_rows: int = None):
    """Times the CPU oracle (quant + W8A8 GEMM) on a bounded row sample."""
    import oracle
    x = wl.make_x()
    w = wl.make_w()
    s, inv = oracle.smooth_factors(x, w)
    q_w, s_ch = oracle.quant_weight(w, s)
    del w
    nt = oracle.threads()

    def run(rows):
        xs = x[:rows].contiguous()
        t0 = time.perf_counter()
        q_a, s_tok = oracle.quant_per_token(xs, inv)
        oracle.w8a8_scaled_mm(q_a, s_tok, q_w, s_ch)
        return time.perf_counter() - t0

    t1 = run(nt)
    rows = max(1, min(wl.M, int(nt * target_s / max(t1, 1e-6))))
    if max_rows:
        rows = min(rows, max_rows)
    return rows, nt, run


def oracle_other_configs(inputs):
    """The CPU oracle timed once on each of the other workloads, in each
    workload's own metric (a bounded row sample where the full workload would
    take more than a few seconds; the sample is stated)."""
    import oracle
    out = []

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    for i in (0, 1):  # tiny and decode W8A8: quant + GEMM, all rows
        wl = inputs.workload(i)
        x, w = wl.make_x(), wl.make_w()
        s, inv = oracle.smooth_factors(x, w)
        q_w, s_ch = oracle.quant_weight(w, s)

        def run():
            q_a, s_tok = oracle.quant_per_token(x, inv)
            oracle.w8a8_scaled_mm(q_a, s_tok, q_w, s_ch)
        t = timed(run)
        byt = algo_bytes_quant(wl.M, wl.K) + algo_bytes_w8a8(wl.M, wl.N, wl.K)
        out.append({"workload": wl.name, "metric": "GB/s (quant + GEMM, algorithmic bytes)",
                    "value": byt / t / 1e9, "unit": "GB/s", "seconds": t,
                    "tops": 2.0 * wl.M * wl.N * wl.K / t / 1e12, "sample": "all rows"})
    wl = inputs.workload(3)  # gs128: a row sample
    x, w = wl.make_x(), wl.make_w()
    q_w, s_blk = oracle.quant_weight(w, None, group=128)
    rows = 256
    q_a, s_tok = oracle.quant_per_token(x[:rows].contiguous(), None)
    t = timed(lambda: oracle.gs128_mm(q_a, s_tok, q_w, s_blk))
    out.append({"workload": wl.name, "metric": "TOPS (gs128 GEMM)",
                "value": 2.0 * rows * wl.N * wl.K / t / 1e12, "unit": "TOPS", "seconds": t,
                "sample": f"first {rows} of {wl.M} token rows, all N columns"})
    wl = inputs.workload(4)  # W8A16 down_proj
    w = wl.make_w()
    q_w, s_ch = oracle.quant_weight(w, None)
    for M in (1, 16):
        x = wl.make_x(M)
        t = timed(lambda: oracle.w8a16_mm(x, q_w, s_ch))
        out.append({"workload": f"{wl.name}_M{M}", "metric": "GB/s (algorithmic bytes)",
                    "value": algo_bytes_w8a16(M, wl.N, wl.K) / t / 1e9, "unit": "GB/s",
                    "seconds": t, "sample": "all rows"})
    return out


def reference_arm(args, peaks):
    ws, rank, _ = dist_info()
    if rank != 0:
        return 0
    from w8a8_int8_quantized_sq_b200 import inputs
    wl = inputs.workload(2)
    # about 0.5 s of oracle work per step, less for long runs: the whole
    # --steps + --warmup run stays near two minutes
    per_step = min(0.5, 120.0 / (args.steps + args.warmup))
    rows, nt, run = oracle_sample(wl, target_s=per_step)
    ops_step = 2.0 * rows * wl.N * wl.K
    for _ in range(args.warmup):
        run(rows)
    t = 0.0
    for _ in range(args.steps):
        t += run(rows)
    value = ops_step * args.steps / t / 1e12
    sample = (f"first {rows} of {wl.M} token rows of {wl.name} per step "
              "(oracle per-token quant + int32 GEMM + epilogue, all N columns)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": wl.name, "M": wl.M, "K": wl.K, "N": wl.N,
                       "rows_per_step": rows},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": nt, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- main arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile", choices=["w8a8", "gs128", "w8a16", "pg128", "fp8", "w8a16g",
                                          "rmsnorm"], default=None,
                    help="run one operation at --M/--N/--K for --steps calls (for ncu)")
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=34816)
    ap.add_argument("--K", type=int, default=5120)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    peaks = load_peaks()
    if args.impl == "reference":
        return reference_arm(args, peaks)
    if args.profile:
        return profile_case(args)

    import w8a8_int8_quantized_sq_b200 as sq
    from w8a8_int8_quantized_sq_b200 import inputs

    world, rank, local = dist_info()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sq.lib()  # fails loudly if the CUDA library is missing

    barrier, max_over_ranks = replica_collectives(world, dev)

    # ---------------- prefill W8A8 (the headline workload)
    wl = inputs.workload(2)
    M, N, K = wl.M, wl.N, wl.K
    x_cpu = wl.make_x()
    x = x_cpu.to(dev)
    w = wl.make_w().to(dev)
    s_sm, inv_s = sq.smooth_factors(x, w)
    q_w, s_ch = sq.quant_weight(w, s_sm)
    del w
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()

    # The dense INT8 (and FP8) tensor rate of this device, measured first,
    # on a cool GPU, with the library's tcgen05 issue-rate probe (burst:
    # about a millisecond per launch); 2 x the measured BF16 matmul is kept
    # beside it for reference.
    int8_probe = sq.mma_peak(sq.PEAK_I8)
    fp8_probe = sq.mma_peak(sq.PEAK_F8)

    # One step = the whole layer through the fused entry point
    # (sq_w8a8_linear: quant, then the GEMM as a programmatic dependent).
    def step():
        sq.linear_w8a8(x, inv_s, q_w, s_ch, out=y)

    for _ in range(args.warmup):
        step()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier()
    sampler.start()
    start.record()
    for _ in range(args.steps):
        step()
    end.record()
    barrier()
    clocks = sampler.result()
    total_s = max_over_ranks(start.elapsed_time(end) * 1e-3)

    # The kernels on their own, live, same inputs: CUDA events around every
    # launch on the launching stream (the GEMM timing is the roofline's).
    n_kernel = max(10, min(args.steps, 100))
    q_a, s_tok = sq.quant_per_token(x, inv_s)
    for _ in range(3):
        sq.w8a8_scaled_mm(q_a, s_tok, q_w, s_ch, out=y)
    evg = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_kernel)]
    barrier()
    for i in range(n_kernel):
        evg[i][0].record()
        sq.w8a8_scaled_mm(q_a, s_tok, q_w, s_ch, out=y)
        evg[i][1].record()
    barrier()
    gemm_s = statistics.mean(e[0].elapsed_time(e[1]) for e in evg) * 1e-3
    # The quant kernel (about 25 us) is shorter than a host launch of the
    # binding, so events around single launches would time the host: time it
    # as a CUDA graph of back-to-back launches on inputs that rotate over more
    # than L2.
    xs = [x] + [x.clone() for _ in range(2)]
    quant_s = time_graph(lambda i: sq.quant_per_token(xs[i % 3], inv_s), 12, reps=3)
    del xs
    ops_step = 2.0 * M * N * K
    value = whole_job_tops(ops_step, args.steps, world, total_s)
    int8_proxy = peaks["bf16_tflops"] * INT8_PER_BF16
    int8_peak = int8_probe if int8_probe > 0 else int8_proxy
    peaks["int8_tops"] = int8_peak
    peaks["fp8_tops"] = fp8_probe if fp8_probe > 0 else int8_peak
    gemm_tops = ops_step / gemm_s / 1e12

    # Sustained: the same step back to back for at least two seconds (the
    # short loop above is a burst that ends before the power cap settles).
    sus_steps = max(args.steps, int(2.0 / max(total_s / args.steps, 1e-6)) + 1)
    sampler = ClockSampler(local)
    barrier()
    sampler.start()
    start.record()
    for _ in range(sus_steps):
        step()
    end.record()
    barrier()
    sus_clocks = sampler.result()
    sus_s = max_over_ranks(start.elapsed_time(end) * 1e-3)
    sus_tops = whole_job_tops(2.0 * M * N * K, sus_steps, world, sus_s)
    sustained = {"value": sus_tops, "unit": "TOPS", "steps": sus_steps, "seconds": sus_s,
                 "ms_per_step": sus_s / sus_steps * 1e3, "clocks": sus_clocks,
                 "tops_per_ghz": (sus_tops / (sus_clocks["sm_mhz"] / 1000.0)
                                  if sus_clocks.get("sm_mhz") else None)}
    # the tensor rate under the same conditions: the probe run back to back
    # for about two seconds right after
    sus_probe = sq.mma_peak(sq.PEAK_I8, iters=1 << 21, launches=8)
    sustained["int8_peak_sustained"] = sus_probe
    sustained["frac_of_sustained_peak"] = sus_tops / sus_probe if sus_probe > 0 else None

    # ---------------- end to end through the public API, host buffers
    e2e_steps = max(3, min(args.steps, 10))
    x_h = x_cpu.pin_memory()
    y_h = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    x_d = torch.empty_like(x)

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        yy = sq.linear_w8a8(x_d, inv_s, q_w, s_ch)
        y_h.copy_(yy, non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(e2e_steps):
        e2e_step()
    b.record()
    barrier()
    e2e_s = max_over_ranks(a.elapsed_time(b) * 1e-3)
    e2e = {"value": whole_job_tops(ops_step, e2e_steps, world, e2e_s), "unit": "TOPS",
           "h2d_bytes_per_step": x_h.numel() * 2, "d2h_bytes_per_step": y_h.numel() * 2,
           "steps": e2e_steps}
    del x_h, y_h, x_d

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_s / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": wl.name, "M": M, "K": K, "N": N,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (q_w 178 MB, x 84 MB, y 570 MB)",
                   "step": "sq_w8a8_linear (per-token quant + W8A8 GEMM, PDL)"},
        "pct_of_int8_nominal": 100.0 * value / world / INT8_NOMINAL_TOPS,
        "burst": {"value": value, "unit": "TOPS", "steps": args.steps,
                  "tops_per_ghz": (value / (clocks["sm_mhz"] / 1000.0)
                                   if clocks.get("sm_mhz") else None)},
        "sustained": sustained,
        "roofline": {"bound": "tensor", "kernel": "gemm2_kernel (W8A8, CTA pairs, 256x256 tiles)",
                     "achieved": gemm_tops, "peak": int8_peak, "unit": "TOPS",
                     "frac": gemm_tops / int8_peak,
                     "peak_source": "measured: tcgen05.mma kind::i8 issue-rate probe (sq_mma_peak, "
                                    "all SMs, burst)",
                     "peak_bf16x2": int8_proxy,
                     "frac_of_bf16x2": gemm_tops / int8_proxy,
                     "traffic": gemm_traffic(),
                     "algorithmic_bytes": algo_bytes_w8a8(M, N, K)},
        "split_ms": {"quant": quant_s * 1e3, "gemm": gemm_s * 1e3,
                     "note": "each kernel timed alone after the step loop: GEMM with events per launch, quant as a CUDA graph of back-to-back launches over 3 input copies"},
        "quant_hbm": {"achieved_gbs": algo_bytes_quant(M, K) / quant_s / 1e9,
                      "peak_gbs": peaks["hbm_gbs"],
                      "frac": algo_bytes_quant(M, K) / quant_s / 1e9 / peaks["hbm_gbs"]},
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,  # per timed step: the quant kernel and the GEMM
        "clocks": clocks,
    }
    del x, q_w, y
    torch.cuda.empty_cache()

    line["measured_peaks"] = {"int8_tops": int8_probe, "fp8_tops": fp8_probe,
                              "int8_tops_sustained": sustained["int8_peak_sustained"],
                              "hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"]}
    if not args.no_variants:
        line["variants"] = variants(sq, inputs, dev, peaks) + variants_next(sq, inputs, dev, peaks)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows, nt, run = oracle_sample(wl, target_s=args.cpu_seconds)
        t = run(rows)
        line["cpu_baseline"] = {
            "value": 2.0 * rows * N * K / t / 1e12, "unit": "TOPS", "cores": nt,
            "kind": "oracle", "seconds": t,
            "sample": f"first {rows} of {M} token rows of {wl.name} (oracle quant + GEMM + "
                      "epilogue over all N columns)",
            "per_config": oracle_other_configs(inputs)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def profile_case(args):
    """One operation at the given sizes, warm-up then --steps timed calls."""
    import w8a8_int8_quantized_sq_b200 as sq
    from w8a8_int8_quantized_sq_b200 import inputs
    dev = torch.device("cuda", 0)
    M, N, K = args.M, args.N, args.K
    x = inputs.gen_x(M, K, inputs.SEED_BASE + 100,
                     inputs.XRecipe(col_count=max(1, K // 100), col_factor=30.0)).to(dev)
    w = inputs.gen_w(N, K, inputs.SEED_BASE + 100).to(dev)
    # enough weight copies, used in turn, that no call finds its weights in L2
    l2 = 126 * 2 ** 20
    copies = max(2, -(-3 * l2 // (N * K)))
    if args.profile == "w8a8":
        s, inv = sq.smooth_factors(x, w)
        q_w, s_ch = sq.quant_weight(w, s)
        q_ws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
        fn = lambda i: sq.linear_w8a8(x, inv, q_ws[i % copies], s_ch)  # noqa: E731
    elif args.profile == "gs128":
        q_w, s_blk = sq.quant_weight(w, None, group=128)
        q_a, s_tok = sq.quant_per_token(x, None)
        q_ws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
        fn = lambda i: sq.w8a8_gs128_mm(q_a, s_tok, q_ws[i % copies], s_blk)  # noqa: E731
    elif args.profile == "pg128":
        q_w, s_blk = sq.quant_weight(w, None, group=128)
        q_a, s_a = sq.quant_per_group(x, None)
        q_ws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
        fn = lambda i: sq.w8a8_pg128_mm(q_a, s_a, q_ws[i % copies], s_blk)  # noqa: E731
    elif args.profile == "fp8":
        q_w, s_w = sq.quant_fp8_block(w)
        q_a, s_a = sq.quant_fp8_per_group(x, None)
        q_ws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
        fn = lambda i: sq.fp8_block_mm(q_a, s_a, q_ws[i % copies], s_w)  # noqa: E731
    elif args.profile == "w8a16g":
        q_w, s_grp = sq.quant_weight(w, None, group=128)
        q_ws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
        fn = lambda i: sq.w8a16_group_mm(x, q_ws[i % copies], s_grp)  # noqa: E731
    elif args.profile == "rmsnorm":
        s, inv = sq.smooth_factors(x, w)
        gamma = sq.fold_norm_weight(w[0].contiguous(), inv)
        xs = [x] + [x.clone() for _ in range(2)]
        fn = lambda i: sq.rmsnorm_quant(xs[i % 3], gamma, 1e-6)  # noqa: E731
    else:
        q_w, s_ch = sq.quant_weight(w, None)
        q_ws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
        fn = lambda i: sq.w8a16_mm(x, q_ws[i % copies], s_ch)  # noqa: E731
    del w
    for i in range(args.warmup):
        fn(i)
    torch.cuda.synchronize()
    t_eager = time_batches(fn, args.steps, warmup=0)
    t_graph = time_graph(fn, args.steps, reps=3)
    print(json.dumps({"profile": args.profile, "M": M, "N": N, "K": K, "steps": args.steps,
                      "weight_copies": copies, "ms_per_call": t_graph * 1e3,
                      "ms_per_call_eager": t_eager * 1e3}),
          flush=True)
    return 0


def variants(sq, inputs, dev, peaks):
    """The other workloads, each timed alone with enough weight copies to exceed L2."""
    out = []
    hbm = peaks["hbm_gbs"]
    l2 = 126 * 2 ** 20

    # decode-shaped W8A8 (M=8): weight-read bound
    wl = inputs.workload(1)
    x = wl.make_x().to(dev)
    w = wl.make_w().to(dev)
    s, inv = sq.smooth_factors(x, w)
    q_w, s_ch = sq.quant_weight(w, s)
    del w
    copies = max(2, -(-3 * l2 // q_w.numel()))
    qws = [q_w.clone() for _ in range(copies)]
    t = time_graph(lambda i: sq.linear_w8a8(x, inv, qws[i % copies], s_ch), 4 * copies)
    q_a, s_tok = sq.quant_per_token(x, inv)
    tg = time_graph(lambda i: sq.w8a8_scaled_mm(q_a, s_tok, qws[i % copies], s_ch), 4 * copies)
    tq = time_graph(lambda i: sq.quant_per_token(x, inv), 4 * copies)
    # the same GEMM calls launched as programmatic dependents of each other
    sq.set_overlap(True)
    try:
        tg_ov = time_graph(lambda i: sq.w8a8_scaled_mm(q_a, s_tok, qws[i % copies], s_ch),
                           4 * copies)
    finally:
        sq.set_overlap(False)
    byt = algo_bytes_quant(wl.M, wl.K) + algo_bytes_w8a8(wl.M, wl.N, wl.K)
    out.append({"workload": wl.name, "metric": "GB/s (quant + GEMM, algorithmic bytes)",
                "value": byt / t / 1e9, "unit": "GB/s", "us_per_call": t * 1e6,
                "frac_of_hbm": byt / t / 1e9 / hbm, "tokens_per_s": wl.M / t,
                "tops": 2.0 * wl.M * wl.N * wl.K / t / 1e12, "weight_copies": copies,
                "gemm_us": tg * 1e6, "quant_us": tq * 1e6,
                "gemm_frac_of_hbm": algo_bytes_w8a8(wl.M, wl.N, wl.K) / tg / 1e9 / hbm,
                "gemm_us_overlap": tg_ov * 1e6,
                "gemm_frac_of_hbm_overlap": algo_bytes_w8a8(wl.M, wl.N, wl.K) / tg_ov / 1e9 / hbm,
                "timing": "CUDA graph of back-to-back calls, rotating weight copies; "
                          "_overlap: with sq_set_overlap(1)"})
    del qws, q_w, x, q_a

    # gs128 W8A8 (M=2048)
    wl = inputs.workload(3)
    x = wl.make_x().to(dev)
    w = wl.make_w().to(dev)
    q_w, s_blk = sq.quant_weight(w, None, group=128)
    del w
    q_a, s_tok = sq.quant_per_token(x, None)
    copies = max(2, -(-3 * l2 // (q_w.numel() + q_a.numel())))
    sets = [(q_a.clone(), q_w.clone()) for _ in range(copies)]
    t = time_graph(lambda i: sq.w8a8_gs128_mm(sets[i % copies][0], s_tok, sets[i % copies][1],
                                              s_blk), 2 * copies)
    tq = time_graph(lambda i: sq.quant_per_token(x, None), 2 * copies)
    ops = 2.0 * wl.M * wl.N * wl.K
    int8_peak = peaks.get("int8_tops", peaks["bf16_tflops"] * INT8_PER_BF16)
    out.append({"workload": wl.name, "metric": "TOPS (gs128 GEMM)", "value": ops / t / 1e12,
                "unit": "TOPS", "us_per_call": t * 1e6, "frac_of_int8_peak": ops / t / 1e12 / int8_peak,
                "tops_incl_quant": ops / (t + tq) / 1e12, "quant_us": tq * 1e6,
                "weight_copies": copies})
    del sets, q_w, q_a, x

    # W8A16 down_proj (K=17408, N=5120), M = 1, 16, 8192
    wl = inputs.workload(4)
    w = wl.make_w().to(dev)
    q_w, s_ch = sq.quant_weight(w, None)
    del w
    copies = max(2, -(-3 * l2 // q_w.numel()))
    qws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
    for M in inputs.W8A16_M_VALUES:
        x = wl.make_x(M).to(dev)
        if M <= 16:
            t = time_graph(lambda i: sq.w8a16_mm(x, qws[i % copies], s_ch), 4 * copies)
            sq.set_overlap(True)
            try:
                t_ov = time_graph(lambda i: sq.w8a16_mm(x, qws[i % copies], s_ch), 4 * copies)
            finally:
                sq.set_overlap(False)
            byt = algo_bytes_w8a16(M, wl.N, wl.K)
            out.append({"workload": f"{wl.name}_M{M}", "metric": "GB/s (algorithmic bytes)",
                        "value": byt / t / 1e9, "unit": "GB/s", "us_per_call": t * 1e6,
                        "frac_of_hbm": byt / t / 1e9 / hbm, "tokens_per_s": M / t,
                        "weight_copies": copies, "us_per_call_overlap": t_ov * 1e6,
                        "frac_of_hbm_overlap": byt / t_ov / 1e9 / hbm,
                        "timing": "CUDA graph of back-to-back calls, rotating weight copies; "
                                  "_overlap: with sq_set_overlap(1)"})
        else:
            t = time_batches(lambda i: sq.w8a16_mm(x, qws[i % 2], s_ch), 10)
            fl = 2.0 * M * wl.N * wl.K
            out.append({"workload": f"{wl.name}_M{M}", "metric": "TFLOP/s (bf16 tensor)",
                        "value": fl / t / 1e12, "unit": "TFLOP/s", "us_per_call": t * 1e6,
                        "frac_of_bf16_peak": fl / t / 1e12 / peaks["bf16_tflops"],
                        "tokens_per_s": M / t})
        del x
    del qws, q_w
    torch.cuda.empty_cache()
    return out


def variants_next(sq, inputs, dev, peaks):
    """The next rows: fused RMSNorm + fold + quantisation, per-group INT8 and
    FP8 activation quantisation, per-group x gs128 and FP8 block GEMMs, and
    group-wise W8A16; each timed alone, inputs rotating over more than L2."""
    out = []
    hbm = peaks["hbm_gbs"]
    l2 = 126 * 2 ** 20

    # prefill hidden state, M=8192 K=5120: the norm / quantisation kernels
    wl = inputs.workload(2)
    M, K = wl.M, wl.K
    x = wl.make_x().to(dev)
    w = wl.make_w().to(dev)
    _, inv = sq.smooth_factors(x, w)
    del w
    w_norm = inputs.gen_w(1, K, inputs.SEED_BASE + 77, sigma=0.1)[0].contiguous().to(dev)
    gamma = sq.fold_norm_weight(w_norm, inv)
    xs = [x, x.clone(), x.clone()]
    for group in (0, 128):
        t = time_graph(lambda i: sq.rmsnorm_quant(xs[i % 3], gamma, 1e-6, group), 12, reps=3)
        nsc = M if group == 0 else M * (K // 128)
        byt = 2 * M * K + 4 * K + M * K + 4 * nsc + 4 * M
        out.append({"workload": f"rmsnorm_quant_M{M}_K{K}_" + ("per_token" if group == 0 else "g128"),
                    "metric": "GB/s (algorithmic bytes)", "value": byt / t / 1e9, "unit": "GB/s",
                    "us_per_call": t * 1e6, "frac_of_hbm": byt / t / 1e9 / hbm,
                    "tokens_per_s": M / t,
                    "timing": "CUDA graph of 12 back-to-back launches over 3 input copies"})
    for name, fn in (("quant_per_group_int8", lambda i: sq.quant_per_group(xs[i % 3], inv)),
                     ("quant_per_group_fp8", lambda i: sq.quant_fp8_per_group(xs[i % 3], inv))):
        t = time_graph(fn, 12, reps=3)
        byt = 2 * M * K + 4 * K + M * K + 4 * M * (K // 128)
        out.append({"workload": f"{name}_M{M}_K{K}", "metric": "GB/s (algorithmic bytes)",
                    "value": byt / t / 1e9, "unit": "GB/s", "us_per_call": t * 1e6,
                    "frac_of_hbm": byt / t / 1e9 / hbm, "tokens_per_s": M / t})
    del xs, x, gamma

    # block-scaled GEMMs at the gs128 workload's shape (M=2048, K=5120, N=5120)
    wl = inputs.workload(3)
    M, N, K = wl.M, wl.N, wl.K
    x = wl.make_x().to(dev)
    w = wl.make_w().to(dev)
    q_w, s_blk = sq.quant_weight(w, None, group=128)
    qf_w, s_w = sq.quant_fp8_block(w)
    del w
    q_a, s_a = sq.quant_per_group(x, None)
    qf_a, sf_a = sq.quant_fp8_per_group(x, None)
    copies = max(2, -(-3 * l2 // (q_w.numel() + q_a.numel())))
    ops = 2.0 * M * N * K
    sets = [(q_a.clone(), q_w.clone()) for _ in range(copies)]
    t = time_graph(lambda i: sq.w8a8_pg128_mm(sets[i % copies][0], s_a, sets[i % copies][1], s_blk),
                   2 * copies)
    out.append({"workload": f"pg128_w8a8_M{M}_K{K}_N{N}", "metric": "TOPS (per-group x gs128 GEMM)",
                "value": ops / t / 1e12, "unit": "TOPS", "us_per_call": t * 1e6,
                "frac_of_int8_peak": ops / t / 1e12 / peaks["int8_tops"], "weight_copies": copies})
    del sets
    sets = [(qf_a.clone(), qf_w.clone()) for _ in range(copies)]
    t = time_graph(lambda i: sq.fp8_block_mm(sets[i % copies][0], sf_a, sets[i % copies][1], s_w),
                   2 * copies)
    out.append({"workload": f"fp8_block_M{M}_K{K}_N{N}", "metric": "TOPS (FP8 block GEMM)",
                "value": ops / t / 1e12, "unit": "TOPS", "us_per_call": t * 1e6,
                "frac_of_fp8_peak": ops / t / 1e12 / peaks["fp8_tops"], "weight_copies": copies})
    del sets, q_w, qf_w, q_a, qf_a, x

    # group-wise W8A16 down_proj (K=17408, N=5120), M = 1, 16, 8192
    wl = inputs.workload(4)
    w = wl.make_w().to(dev)
    q_w, s_grp = sq.quant_weight(w, None, group=128)
    del w
    copies = max(2, -(-3 * l2 // q_w.numel()))
    qws = [q_w] + [q_w.clone() for _ in range(copies - 1)]
    for M in inputs.W8A16_M_VALUES:
        x = wl.make_x(M).to(dev)
        if M <= 16:
            t = time_graph(lambda i: sq.w8a16_group_mm(x, qws[i % copies], s_grp), 4 * copies)
            byt = 2 * M * wl.K + wl.N * wl.K + 4 * wl.N * (wl.K // 128) + 2 * M * wl.N
            out.append({"workload": f"w8a16_group_K{wl.K}_N{wl.N}_M{M}",
                        "metric": "GB/s (algorithmic bytes)", "value": byt / t / 1e9,
                        "unit": "GB/s", "us_per_call": t * 1e6, "frac_of_hbm": byt / t / 1e9 / hbm,
                        "tokens_per_s": M / t, "weight_copies": copies})
        else:
            t = time_batches(lambda i: sq.w8a16_group_mm(x, qws[i % 2], s_grp), 10)
            fl = 2.0 * M * wl.N * wl.K
            out.append({"workload": f"w8a16_group_K{wl.K}_N{wl.N}_M{M}",
                        "metric": "TFLOP/s (bf16 tensor)", "value": fl / t / 1e12,
                        "unit": "TFLOP/s", "us_per_call": t * 1e6,
                        "frac_of_bf16_peak": fl / t / 1e12 / peaks["bf16_tflops"],
                        "tokens_per_s": M / t})
        del x
    del qws, q_w
    torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    sys.exit(main())
