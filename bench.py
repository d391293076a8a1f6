#!/usr/bin/env python
"""Benchmark of the per-group low-bit quantized linear hot path on B200.

One step = the whole hot path over the FLUX-like DiT linears (4-bit, group 128, rank-32
bf16 branch, bias, M = 4096 tokens): for each of W 3072x3072, 12288x3072 and 3072x12288,
quantize + pack the residual weights (one wq_quantize_pack_many call for the three), then
run the fused dequant-GEMM y = x deq(R)^T + (x L1) L2 + bias (wq_linear) of each.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). `value` is the dequant-GEMM throughput of the whole step
(algorithmic GEMM FLOPs of all ranks / device time of the step, max over ranks), in TFLOP/s.
Multi-GPU runs are independent replicas (the path has no exchange step): weak scaling.
`--impl reference` times the CPU oracle (the only baseline for this method) on a bounded
sample of the same workload.
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

METRIC = "dequant-GEMM TFLOP/s & weight GB/s (% roofline); quantize+pack Gparam/s"
WORKLOAD = ("FLUX-like DiT linears W 3072x3072, 12288x3072, 3072x12288; M=4096 tokens; "
            "4-bit per-group(128); rank-32 bf16 low-rank branch; bias; step = quantize+pack + dequant-GEMM")
BITS, RANK, M_TOKENS = 4, 32, 4096
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_flops(N, K, M, rank):
    return 2.0 * M * N * K + 2.0 * M * rank * (K + N)


def weight_bytes(N, K, bits):
    return N * K * bits / 8 + N * K / 128 * 4


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML from a background thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = str(e)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "nvml")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workload

def make_workload(device):
    """Seeded synthetic FLUX-like linears, resident on `device`, plus their host copies."""
    import numpy as np
    import torch
    from bit_weight_quantization_wq_b200 import synth

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    lins = synth.flux_linears(M=M_TOKENS, rank=RANK)
    out = []
    for lin in lins:
        N, K = lin["N"], lin["K"]
        d = dict(N=N, K=K, host=lin,
                 R=dev(lin["R"]), x=dev(lin["x"]), L1=dev(lin["L1"]), L2=dev(lin["L2"]), bias=dev(lin["bias"]),
                 packed=torch.empty((N, K * BITS // 8), dtype=torch.uint8, device=device),
                 scales=torch.empty((N, K // 128), dtype=torch.float32, device=device),
                 y=torch.empty((M_TOKENS, N), dtype=torch.bfloat16, device=device))
        out.append(d)
    return out


def run_step(wq, lins, ws, pack, events=None):
    """One step: quantize + pack the three residuals (one prepared wq_quantize_pack_many
    call, a single launch), then the three quantized linears. events: [pack start, pack end,
    end of linear 0, 1, 2]."""
    if events is not None:
        events[0].record()
    pack()
    if events is not None:
        events[1].record()
    for i, d in enumerate(lins):
        wq.wq_linear(d["x"], d["packed"], d["scales"], BITS, d["N"], L1=d["L1"], L2=d["L2"],
                     bias=d["bias"], y=d["y"], workspace=ws)
        if events is not None:
            events[2 + i].record()


# ----------------------------------------------------------------------------- recorded traffic

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per wq_linear call of the step
# (prepass + tensor-core kernel, mean over the 3 shapes), recorded from one ncu capture of
# this workload, keyed by a digest of the kernel sources it was taken on; a changed kernel
# reports null until it is captured again.
RECORDED_TRAFFIC = {
    # 57.0, 131.2 and 248.9 MB for 3072x3072, 12288x3072 and 3072x12288 (N x K)
    "873ace71abbc1ec1": 145.69e6,
}
KERNEL_SOURCES = ("gemm_tc.cuh", "unpack.cuh", "common.cuh", "wq_api.cu")


def kernel_source_digest() -> str:
    import hashlib
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bit_weight_quantization_wq_b200", "csrc")
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    return RECORDED_TRAFFIC.get(kernel_source_digest())


# ----------------------------------------------------------------------------- oracle legs

def oracle_sample(lins_host, rows_per_linear: int, pack_rows: int):
    """Run the CPU oracle on a bounded sample: quantize + pack `pack_rows` weight rows of each
    residual, dequantize those rows, and evaluate the fp64 linear for `rows_per_linear` token
    rows against them (scaled to the full output width). Returns (flops, params, seconds)."""
    import numpy as np
    import oracle
    flops = params = 0.0
    t0 = time.perf_counter()
    for i, lin in enumerate(lins_host):
        N, K = lin["N"], lin["K"]
        n = min(pack_rows, N)
        codes, scales = oracle.quantize(lin["R"][:n], BITS)
        oracle.pack(codes, BITS)
        deq = oracle.dequant(codes, scales, BITS)
        rows = (np.arange(rows_per_linear, dtype=np.int64) + 17 * i) % lin["x"].shape[0]
        oracle.linear_rows(lin["x"], deq, lin["L1"], lin["L2"][:, :n], lin["bias"][:n], rows)
        flops += gemm_flops(n, K, rows_per_linear, RANK)
        params += n * K
    return flops, params, time.perf_counter() - t0


def cpu_baseline(lins_host, budget_s: float = 12.0):
    import oracle
    prow = min(lin["N"] for lin in lins_host)
    # calibration: the sample costs a fixed quantize+pack part plus a per-token-row part
    _, _, t8 = oracle_sample(lins_host, 8, prow)
    _, _, t40 = oracle_sample(lins_host, 40, prow)
    per_row = max((t40 - t8) / 32, 1e-5)
    fixed = max(t8 - 8 * per_row, 0.0)
    rows = int(max(8, min(4096, (budget_s - fixed) / per_row)))
    f, p, t = oracle_sample(lins_host, rows, prow)
    return {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": (f"C oracle (fp32 quantize+pack, fp64 linear with the rank-32 branch) on {prow} weight rows "
                       f"of each of the 3 residuals x {rows} token rows: {f / 1e9:.2f} GFLOP in {t:.1f} s "
                       f"(pack+dequant+linear wall time)")}


def reference_arm(args):
    """--impl reference: the CPU oracle timed on bounded samples of the workload."""
    world, rank, _ = dist_info()
    if rank != 0:
        return 0
    import oracle
    from bit_weight_quantization_wq_b200 import synth
    lins_host = synth.flux_linears(M=M_TOKENS, rank=RANK)
    steps, warmup = args.steps, args.warmup
    f, p, t = oracle_sample(lins_host, 2, 256)
    per_step = max(1.0, min(20.0, 90.0 / max(1, steps + warmup)))
    scale = max(1.0, per_step / max(t, 1e-3))
    rows, prow = max(2, min(256, int(2 * scale))), max(128, min(3072, int(256 * scale)))
    for _ in range(warmup):
        oracle_sample(lins_host, rows, prow)
    tot_f = tot_t = 0.0
    for _ in range(steps):
        f, p, t = oracle_sample(lins_host, rows, prow)
        tot_f += f
        tot_t += t
    value = tot_f / tot_t / 1e12 if tot_t > 0 else 0.0
    sample = (f"per step: C oracle on {prow} weight rows of each of the 3 residuals x {rows} token rows "
              f"({tot_f / max(steps, 1) / 1e9:.2f} GFLOP)")
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps,
            "warmup": warmup, "ms_per_step": 1e3 * tot_t / max(steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "kind": "oracle", "cores": oracle.num_threads(),
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- main arm

def main_arm(args):
    import torch
    import bit_weight_quantization_wq_b200 as wq
    from bit_weight_quantization_wq_b200 import build as wq_build

    world, rank, local = dist_info()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    if rank == 0:
        wq_build.build()
    barrier(world, device)
    wq.lib()

    lins = make_workload(device)
    ws = torch.empty(max(wq.wq_linear_workspace_bytes(M_TOKENS, d["N"], d["K"], BITS, RANK) for d in lins),
                     dtype=torch.uint8, device=device)
    step_flops = sum(gemm_flops(d["N"], d["K"], M_TOKENS, RANK) for d in lins)
    step_params = sum(d["N"] * d["K"] for d in lins)
    step_wbytes = sum(weight_bytes(d["N"], d["K"], BITS) for d in lins)

    pack = wq.PackJobs([(d["R"], BITS, d["packed"], d["scales"]) for d in lins])
    for _ in range(args.warmup):
        run_step(wq, lins, ws, pack)
    torch.cuda.synchronize()
    if wq.wq_device_status() != 0:
        raise RuntimeError("device status not clean after warm-up")

    # ---------------------------------------------------------------- timed region
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 + len(lins))] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    launches0 = wq.wq_launch_count()
    with ClockSampler(device.index) as clocks:
        start.record()
        for k in range(K):
            run_step(wq, lins, ws, pack, ev[k])
        stop.record()
        torch.cuda.synchronize()
    launches = wq.wq_launch_count() - launches0
    barrier(world, device)
    step_ms = start.elapsed_time(stop) / K
    step_ms = max_over_ranks(step_ms, world, device)
    pack_ms = sum(ev[k][0].elapsed_time(ev[k][1]) for k in range(K)) / K
    lin_ms = sum(ev[k][1].elapsed_time(ev[k][-1]) for k in range(K)) / K
    if wq.wq_device_status() != 0:
        raise RuntimeError("device status not clean after the timed region")

    peaks, peak_src = load_peaks()
    lin_tflops = step_flops / (lin_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": lin_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": lin_tflops / peaks["bf16_tflops"], "traffic": recorded_traffic(),
                "traffic_source": "recorded: ncu dram__bytes_read.sum + dram__bytes_write.sum per call, "
                                  "same workload and kernel sources (null when the kernel changed since)",
                "kernel": "wq_linear (lowrank_prepass_kernel + tc_linear_kernel<4>), mean over the 3 shapes",
                "peak_source": f"{peak_src} bf16 dense (burst)"}

    # ---------------------------------------------------------------- e2e through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = e2e_leg(wq, lins, ws, args, device, world, step_flops)

    value = step_flops * world / (step_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_tokens": M_TOKENS * world, "bits": BITS, "group": 128,
                   "rank": RANK, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: a step reads ~320 MB of distinct inputs, so each kernel's "
                         "operands were evicted by the rest of the step before it runs again"},
        "roofline": roofline,
        "breakdown": {
            "linear_ms_per_step": lin_ms, "pack_ms_per_step": pack_ms,
            "linear_tflops": lin_tflops,
            "linear_weight_gbs": step_wbytes / (lin_ms * 1e-3) / 1e9,
            "pack_gparams": step_params / (pack_ms * 1e-3) / 1e9,
            "pack_gbs": (2 * step_params + step_wbytes) / (pack_ms * 1e-3) / 1e9,
            "pack_hbm_frac": (2 * step_params + step_wbytes) / (pack_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        },
        "clocks": clocks.summary(),
        "gpu_launches": launches,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_legs:
        line["breakdown"].update(breakdown_legs(wq, device, peaks))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline([d["host"] for d in lins], budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def _l2_flusher(device):
    """Write then read a 256 MB buffer (twice the 126 MB L2) so the next call starts cold."""
    import torch
    flush = torch.empty(32 << 20, dtype=torch.int64, device=device)
    sink = torch.empty((), dtype=torch.int64, device=device)

    def f():
        flush.fill_(1)
        torch.sum(flush, dim=0, out=sink)
    return f


def _time_calls(run, reps, flush=None, warmup=3):
    """Median device time (us) of `run`, each call bracketed by its own CUDA events on the
    current stream, optionally with L2 flushed before it (outside the events)."""
    import torch
    for _ in range(warmup):
        if flush:
            flush()
        run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        if flush:
            flush()
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)
    return t[len(t) // 2]


def _time_graph(calls, reps=5):
    """Per-call device time (us) of a list of calls captured back to back in one CUDA graph
    and replayed `reps` times (CUDA events around the replays): launch-to-launch time with no
    host work and no other kernel between the calls."""
    import torch
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        for c in calls:
            c()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st):
        for c in calls:
            c()
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    del graph
    return a.elapsed_time(b) * 1e3 / (reps * len(calls))


def breakdown_legs(wq, device, peaks, stack_blocks=40, model_blocks=49):
    """The parts of the metric beyond the step, each timed on the device (CUDA events):

    small_m     weight GB/s and HBM fraction of the Wan-like 13824x5120 and 5120x5120 linears
                at 1 and 16 tokens, 4 and 5 bits: a CUDA graph of back-to-back calls over
                enough distinct weight copies (> 400 MB) that no call finds its weight in L2;
    m128        the 128-token crossover of the same shapes at 4 bits, timed the same way,
                against whichever roofline bound binds (max of FLOPs at the bf16 peak and
                bytes at HBM);
    stack       the mixed-precision 40-block DiT stack: 4096 tokens through all 400 linears in
                order (each output is the next input), TFLOP/s of a whole pass;
    model       whole-model quantize+pack: all 490 tensors of the 49-block model resident
                (34.4 GB bf16), one wq_quantize_pack_many call, Gparam/s and packed size; the
                error table of all of them at every width (wq_quant_error_many), each tensor's
                SNR at its width, and the per-tensor width search at 5.0 bits per weight.
    Weights are seeded device draws of the workloads' recipe."""
    import numpy as np
    import torch
    from bit_weight_quantization_wq_b200 import synth
    hbm, bf16, bf16_s = peaks["hbm_gbs"], peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    out = {}
    # ------------------------------------------------------------ small M and the crossover
    small, cross = [], []
    for si, (N, K) in enumerate(synth.WAN_SHAPES):
        for bits in (4, 5):
            W = synth.weight_torch(synth.torch_generator(3, si, 0), N, K, 0.015)
            packed, scales = wq.wq_quantize_pack(W, bits)
            del W
            copies = max(4, int(400e6 // (packed.numel() + 4 * scales.numel())) + 1)
            ws = [(packed.clone(), scales.clone()) for _ in range(copies)]
            b = (torch.randn(N, device=device) * 0.01).to(torch.bfloat16)
            for M in ((1, 16, 128) if bits == 4 else (1, 16)):
                x = torch.randn(M, K, device=device).to(torch.bfloat16)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                calls = [lambda p=p, sc=sc: wq.wq_linear(x, p, sc, bits, N, bias=b, y=y) for p, sc in ws]
                us = _time_graph(calls)
                wbytes = weight_bytes(N, K, bits)
                nbytes = wbytes + 2 * M * K + 2 * M * N + 2 * N
                flops = gemm_flops(N, K, M, 0)
                rec = {"shape": f"{N}x{K}", "M": M, "bits": bits, "us": us,
                       "weight_gbs": wbytes / us / 1e3, "tflops": flops / us / 1e6}
                if M <= 16:
                    rec["hbm_frac"] = nbytes / us / 1e3 / hbm
                    small.append(rec)
                else:
                    t_roof = max(flops / (bf16 * 1e12), nbytes / (hbm * 1e9)) * 1e6
                    rec["bound"] = "tensor" if flops / (bf16 * 1e12) > nbytes / (hbm * 1e9) else "hbm"
                    rec["roofline_us"] = t_roof
                    rec["frac"] = t_roof / us
                    cross.append(rec)
            del ws
    rot = "inputs larger than L2: each call's weight is one of >400 MB of distinct copies, calls back to back in a CUDA graph"
    out["small_m"] = {"l2": rot, "peak_hbm_gbs": hbm, "cases": small}
    out["m128"] = {"l2": rot, "cases": cross}
    torch.cuda.empty_cache()
    # ------------------------------------------------------------ 40-block stack (config 4)
    layers = []
    for blk in range(stack_blocks):
        widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=4, block=blk)
        Ws = [synth.weight_torch(synth.torch_generator(4, blk, i), N, K, 0.015)
              for i, (N, K) in enumerate(synth.BLOCK_SHAPES)]
        outs = wq.PackJobs(list(zip(Ws, widths)))()
        for (N, K), bits, (p, sc) in zip(synth.BLOCK_SHAPES, widths, outs):
            layers.append((N, K, bits, p, sc))
        del Ws
    Mt = 4096
    x0 = torch.randn(Mt, 5120, device=device).to(torch.bfloat16)
    bufs = {5120: [torch.empty((Mt, 5120), dtype=torch.bfloat16, device=device) for _ in range(2)],
            13824: [torch.empty((Mt, 13824), dtype=torch.bfloat16, device=device)]}

    def stack_pass():
        cur, k = x0, 0
        for N, K, bits, p, sc in layers:
            ys = bufs[N]
            y = ys[k % len(ys)]
            k += 1
            wq.wq_linear(cur, p, sc, bits, N, y=y)
            cur = y

    stack_flops = sum(gemm_flops(N, K, Mt, 0) for N, K, _, _, _ in layers)
    us = _time_calls(stack_pass, 3, None, warmup=2)
    tf = stack_flops / us / 1e6
    out["stack"] = {"blocks": stack_blocks, "linears": len(layers), "tokens": Mt, "ms_per_pass": us / 1e3,
                    "tflops": tf, "frac_bf16_sustained": tf / bf16_s, "frac_bf16_burst": tf / bf16,
                    "bits_histogram": {str(b): sum(1 for l in layers if l[2] == b) for b in range(3, 8)},
                    "l2": "inputs larger than L2 (8.8 GB of packed weights per pass)"}
    del layers, bufs, x0
    torch.cuda.empty_cache()
    # ------------------------------------------------------------ 49-block model pack (config 5)
    jobs = []
    for blk in range(model_blocks):
        widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=5, block=blk)
        for i, ((N, K), bits) in enumerate(zip(synth.BLOCK_SHAPES, widths)):
            jobs.append((synth.weight_torch(synth.torch_generator(5, blk, i), N, K, 0.015), bits))
    call = wq.PackJobs(jobs)
    l0 = wq.wq_launch_count()
    call()
    launches = wq.wq_launch_count() - l0
    us = _time_calls(call, 5, None, warmup=2)
    params = sum(W.numel() for W, _ in jobs)
    packed_b = sum(p.numel() + 4 * sc.numel() for p, sc in call.outputs)
    nbytes = 2 * params + packed_b
    out["model"] = {"blocks": model_blocks, "tensors": len(jobs), "params": params, "ms_per_call": us / 1e3,
                    "gparams": params / us / 1e3, "gbs": nbytes / us / 1e3, "hbm_frac": nbytes / us / 1e3 / hbm,
                    "bf16_gb": 2 * params / 1e9, "packed_gb": packed_b / 1e9, "launches_per_call": launches,
                    "l2": "inputs larger than L2 (34 GB of weights per call)"}
    # error table of all 490 tensors at every width (one wq_quant_error_many call), each
    # tensor's SNR at its width, and the per-tensor width search at 5.0 bits per weight
    Ws = [W for W, _ in jobs]
    widths = np.array([b for _, b in jobs])
    table = torch.empty((len(Ws), 6), dtype=torch.float64, device=device)
    err_call = lambda: wq.wq_quant_error_many(Ws, out=table)
    us_err = _time_calls(err_call, 3, None, warmup=1)
    tab = table.cpu().numpy()
    n_w = np.array([W.numel() for W in Ws], np.int64)
    sse_at = tab[np.arange(len(Ws)), widths - 3]
    snr = 10.0 * np.log10(tab[:, 5] / sse_at)
    mse = tab[:, :5] / n_w[:, None]
    t_init = np.random.default_rng(5).standard_normal((15, len(Ws))) * 0.5
    pd_bits, pd_mse, pd_bpw, _ = wq.wq_pd_search(mse, n_w, [3, 4, 5, 6, 7], 5.0, t_init)
    tot = lambda b: float(np.sum(n_w * mse[np.arange(len(Ws)), np.asarray(b) - 3]) / n_w.sum())
    out["model"].update({
        "snr_db": {"mean": float(snr.mean()), "min": float(snr.min()), "max": float(snr.max()),
                   "by_bits": {str(b): float(snr[widths == b].mean()) for b in range(3, 8) if (widths == b).any()}},
        "error_table_ms": us_err / 1e3, "error_table_gparams": params / us_err / 1e3,
        "pd_search_5bpw": {"bpw": pd_bpw, "mse": pd_mse, "mse_uniform_5": tot(np.full(len(Ws), 5)),
                           "mse_histogram_widths": tot(widths),
                           "histogram": {str(b): int((pd_bits == b).sum()) for b in range(3, 8)}}})
    del jobs, call, Ws, table
    torch.cuda.empty_cache()
    return out


def e2e_leg(wq, lins, ws, args, device, world, step_flops):
    """Same metric through the public API with HOST buffers: every step copies its inputs
    from pinned host memory and reads the outputs back, pipelined the way a caller overlaps
    them: host-to-device copies on one stream, the quantize+pack and linear calls on a
    second, device-to-host copies on a third, with double-buffered device inputs and
    outputs so that the copies of one linear overlap the computation of its neighbours."""
    import numpy as np
    import torch
    keys = ("R", "x", "L1", "L2", "bias")
    host_in, host_out = [], []
    for d in lins:
        h = d["host"]
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
        host_in.append({k: pin(h[k]) for k in keys})
        host_out.append(torch.empty((M_TOKENS, d["N"]), dtype=torch.bfloat16).pin_memory())
    h2d = sum(t.numel() * 2 for hi in host_in for t in hi.values())
    d2h = sum(t.numel() * 2 for t in host_out)
    # two device copies of every input and output: buffer b serves linear uses q with q % 2 == b
    dev_in = [[{k: torch.empty_like(d[k]) for k in keys} for _ in range(2)] for d in lins]
    dev_y = [[torch.empty_like(d["y"]) for _ in range(2)] for d in lins]
    s_in, s_comp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in_ready = [[torch.cuda.Event() for _ in range(2)] for _ in lins]
    ev_in_free = [[torch.cuda.Event() for _ in range(2)] for _ in lins]
    ev_out_ready = [[torch.cuda.Event() for _ in range(2)] for _ in lins]
    ev_out_free = [[torch.cuda.Event() for _ in range(2)] for _ in lins]
    use = [0]

    def step():
        for i, (d, hi, ho) in enumerate(zip(lins, host_in, host_out)):
            b = use[0] % 2
            buf, y = dev_in[i][b], dev_y[i][b]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_in_free[i][b])
                for k in keys:
                    buf[k].copy_(hi[k], non_blocking=True)
                ev_in_ready[i][b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in_ready[i][b])
                s_comp.wait_event(ev_out_free[i][b])
                wq.wq_quantize_pack(buf["R"], BITS, packed=d["packed"], scales=d["scales"], stream=s_comp)
                wq.wq_linear(buf["x"], d["packed"], d["scales"], BITS, d["N"], L1=buf["L1"], L2=buf["L2"],
                             bias=buf["bias"], y=y, workspace=ws, stream=s_comp)
                ev_in_free[i][b].record(s_comp)
                ev_out_ready[i][b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_out_ready[i][b])
                ho.copy_(y, non_blocking=True)
                ev_out_free[i][b].record(s_out)
        use[0] += 1

    steps = max(3, min(args.steps, 20))
    for ev_list in (ev_in_free, ev_out_free):          # all buffers start free
        for evs in ev_list:
            for e in evs:
                e.record(torch.cuda.current_stream(device))
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    start.record(s_in)
    s_comp.wait_stream(s_in)
    s_out.wait_stream(s_in)
    for _ in range(steps):
        step()
    # the last device-to-host copy ends the step sequence; wait for the other streams too
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    stop.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop) / steps, world, device)
    return {"value": step_flops * world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "h2d / compute / d2h on three streams, double-buffered device inputs and outputs"}


def case_arm(args):
    """--case: time one call shape (for kernel timing and ncu captures).

    pack:N,K,bits            quantize+pack of an N x K weight
    linear:M,N,K,bits,rank   quantized linear (bias included), path from --path
    model:BLOCKS             quantize+pack of BLOCKS DiT blocks (10 tensors each, mixed widths), one
                             wq_quantize_pack_many call
    model_per_tensor:BLOCKS  the same tensors, one wq_quantize_pack call each
    Inputs are seeded torch draws on the GPU (weights ~N(0, 0.02^2), x ~N(0, 1)).
    """
    import torch
    import bit_weight_quantization_wq_b200 as wq
    from bit_weight_quantization_wq_b200 import build as wq_build
    wq_build.build()
    kind, _, spec = args.case.partition(":")
    vals = [int(v) for v in spec.split(",")]
    g = torch.Generator(device="cuda").manual_seed(1234)
    dev = torch.device("cuda")
    if kind == "pack":
        N, K, bits = vals
        W = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
        packed = torch.empty((N, K * bits // 8), dtype=torch.uint8, device=dev)
        scales = torch.empty((N, K // 128), dtype=torch.float32, device=dev)
        run = lambda: wq.wq_quantize_pack(W, bits, packed=packed, scales=scales)
        work = {"params": N * K, "bytes": 2 * N * K + N * K * bits / 8 + N * K / 32}
    elif kind == "linear":
        M, N, K, bits, rank = vals
        W = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        b = (torch.randn(N, device=dev, generator=g) * 0.01).to(torch.bfloat16)
        L1 = L2 = None
        if rank:
            L1 = (torch.randn(K, rank, device=dev, generator=g) * 0.05).to(torch.bfloat16)
            L2 = (torch.randn(rank, N, device=dev, generator=g) * 0.05).to(torch.bfloat16)
        packed, scales = wq.wq_quantize_pack(W, bits)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, wq.wq_linear_workspace_bytes(M, N, K, bits, rank)), dtype=torch.uint8, device=dev)
        run = lambda: wq.wq_linear(x, packed, scales, bits, N, L1=L1, L2=L2, bias=b, y=y, workspace=ws, path=args.path)
        work = {"flops": gemm_flops(N, K, M, rank), "weight_bytes": weight_bytes(N, K, bits),
                "bytes": 2 * M * K + 2 * M * N + weight_bytes(N, K, bits) + 2 * rank * (K + N) + 2 * N}
    elif kind in ("model", "model_per_tensor"):
        # whole-model quantize+pack: `blocks` DiT blocks of 8 x 5120x5120, 13824x5120 and
        # 5120x13824 tensors, widths drawn i.i.d. from the mixed-precision histogram; every
        # tensor distinct and resident (34 GB at 49 blocks), so each read comes from HBM
        from bit_weight_quantization_wq_b200 import synth
        (blocks,) = vals
        tensors = []
        for blk in range(blocks):
            widths = synth.mixed_bits(len(synth.BLOCK_SHAPES), config=5, block=blk)
            for (N, K), bits in zip(synth.BLOCK_SHAPES, widths):
                W = torch.randn(N, K, device=dev, generator=g, dtype=torch.bfloat16) * 0.015
                tensors.append((W, bits, torch.empty((N, K * bits // 8), dtype=torch.uint8, device=dev),
                                torch.empty((N, K // 128), dtype=torch.float32, device=dev)))

        if kind == "model":
            run = wq.PackJobs(tensors)              # one prepared call: a few launches per width
        else:
            def run():                              # one wq_quantize_pack call per tensor
                for W, bits, packed, scales in tensors:
                    wq.wq_quantize_pack(W, bits, packed=packed, scales=scales)
        params = sum(W.numel() for W, _, _, _ in tensors)
        packed_b = sum(p.numel() + 4 * sc.numel() for _, _, p, sc in tensors)
        work = {"params": params, "bytes": 2 * params + packed_b, "bf16_gb": 2 * params / 1e9,
                "packed_gb": packed_b / 1e9, "tensors": len(tensors)}
    else:
        raise SystemExit(f"unknown case kind {kind!r}")
    # Each timed call starts with a cold L2: a 256 MB buffer (larger than the 126 MB L2) is
    # written and then read before it, outside its events, so L2 holds only clean lines of
    # that buffer (no write-back of dirty lines lands inside the timed call). The flush also
    # keeps the GPU busy while the host queues the call, so host overhead stays out of the
    # events.
    flush = torch.empty(32 << 20, dtype=torch.int64, device=dev)      # 256 MB
    sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2():
        flush.fill_(1)
        torch.sum(flush, dim=0, out=sink)

    for _ in range(max(3, args.warmup)):
        flush_l2()
        run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for s_ev, e_ev in evs:
        flush_l2()
        s_ev.record()
        run()
        e_ev.record()
    torch.cuda.synchronize()
    times = sorted(s_ev.elapsed_time(e_ev) * 1e3 for s_ev, e_ev in evs)
    us = sum(times) / len(times)
    out = {"case": args.case, "path": args.path, "us_per_call": us, "us_min": times[0],
           "us_median": times[len(times) // 2], "l2": "flushed before each call",
           "status": wq.wq_device_status()}
    peaks, src = load_peaks()
    if "flops" in work:
        out["tflops"] = work["flops"] / us / 1e6
        out["weight_gbs"] = work["weight_bytes"] / us / 1e3
        out["frac_bf16"] = out["tflops"] / peaks["bf16_tflops"]
        out["frac_hbm"] = work["bytes"] / us / 1e3 / peaks["hbm_gbs"]
    else:
        out["gparams"] = work["params"] / us / 1e3
        out["gbs"] = work["bytes"] / us / 1e3
        out["frac_hbm"] = out["gbs"] / peaks["hbm_gbs"]
        for k in ("bf16_gb", "packed_gb", "tensors"):
            if k in work:
                out[k] = work[k]
    out["peak_source"] = src
    print(json.dumps(out), flush=True)
    return 0


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-legs", action="store_true", help="skip the small-M / crossover / stack / model legs")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--case", default=None,
                    help="time one shape: pack:N,K,bits, linear:M,N,K,bits,rank, model:BLOCKS or model_per_tensor:BLOCKS")
    ap.add_argument("--path", default="auto", choices=["auto", "small_m", "tensor"], help="kernel family for --case linear")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)
    if args.case:
        return case_arm(args)
    return main_arm(args)


if __name__ == "__main__":
    sys.exit(main())
