"""Benchmark: forward + backward of the Megatron-style tensor-parallel GPT layer on B200.

Default workload: the h=4096 layer (32 heads of 128, ffn 11008, seq 2048, micro-batch 1,
logical tp_size 2, bf16 with fp32 accumulation), synthetic seeded inputs. One "step" = one
mgt_layer_fwd + one mgt_layer_bwd over one batch. With --gpus N (launched by torchrun) every
rank runs its own replica on its own batch (data parallel, no collective on the data path):
weak scaling, value = tokens of all ranks / max-over-ranks time.

Prints ONE JSON line (rank 0). --impl reference times the fp64 CPU oracle instead, on a bounded
sample of the same workload, on this host's cores. --impl torch times the same layer in eager
PyTorch on the GPU (cuBLAS + flash SDPA), as context.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "layer fwd+bwd tokens/s and TFLOP/s (fraction of B200 bf16 peak) at h=4096"
DEFAULT_WORKLOAD = "gpt-h4096-tp2-bf16"
NOMINAL_BF16_TFLOPS = 2250.0
# timed regions shorter than this run at boost clock (burst peak); longer ones are power-capped
BURST_REGION_MS = 1000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# kernels per launch of each profiled family (the C ABI times families, some launch several)
KERNELS_PER_LAUNCH = {"gemm_tc": 1, "gemm_simt": 1, "attn_fwd": 1, "attn_bwd": 2, "ln_fwd": 1,
                      "ln_bwd": 2, "colsum": 1}


GEMM_SOURCES = ("csrc/gemm_tc.cu", "csrc/mgt_device.cuh", "csrc/mgt_internal.h")
GEMM_TRAFFIC = os.path.join(ROOT, "profiles", "gemm_tc_dram_h4096.md")


def gemm_traffic(cfg_name):
    """Average DRAM bytes per GEMM launch from the committed ncu summary, for the workload it
    was captured on and only while the GEMM sources still hash to what was captured."""
    import hashlib
    if cfg_name != DEFAULT_WORKLOAD or not os.path.exists(GEMM_TRAFFIC):
        return None, "no capture for this workload"
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "tensor_transformer_layer_megatron_b200", f), "rb") as fh:
            h.update(fh.read())
    vals = {}
    for line in open(GEMM_TRAFFIC):
        if ":" in line and line.split(":")[0] in ("traffic_bytes_per_launch", "sources_sha256"):
            k, v = line.split(":", 1)
            vals[k] = v.strip()
    if vals.get("sources_sha256") != h.hexdigest():
        return None, "GEMM sources changed since the ncu capture"
    return int(vals["traffic_bytes_per_launch"]), "ncu dram__bytes_read.sum + dram__bytes_write.sum, " \
        "average over the 12 GEMM launches of one step (profiles/gemm_tc_dram_h4096.md)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: d[k] for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock, power and throttle reasons polled through NVML every 5 ms while the timed
    region runs (the host thread waits in the final synchronize meanwhile)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.running = False
        self.th = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[0].isdigit() else self.gpu
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - no NVML: report no clocks
            self.nv = None
            return
        self.running = True
        self.th = threading.Thread(target=self._loop, daemon=True)
        self.th.start()

    def _loop(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while self.running:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0,
                                     int(get_reasons(self.h))))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def stop(self):
        if self.th is None:
            return None
        self.running = False
        self.th.join(timeout=2)
        if not self.samples:
            return None
        sm = sorted(s[0] for s in self.samples)
        reasons = set()
        for _, _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz,
                "power_w_max": round(max(s[1] for s in self.samples), 1),
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(ms, world, device):
    """The job's time is the slowest rank's: all-reduce MAX of this rank's device-timed ms."""
    if world == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, ms_total, steps):
    """Whole-job tokens/s (all ranks' tokens over the max-over-ranks time) and ms per step."""
    ms_step = ms_total / steps
    return tokens_per_rank * world / (ms_step / 1e3), ms_step


def e2e_steps(run, host, steps, stream, graph=True):
    """K steps through the C ABI with host buffers; returns the device-timed ms. Every step
    copies its own x, dy from pinned host memory and its y, dx back. The device buffers are
    double-buffered and the copies run on two copy streams, so step i+1's inputs arrive and
    step i-1's results leave while step i computes (a training loop with prefetch). Within a
    step the forward waits only for x and the backward for dy, and y leaves while the backward
    runs, so only the first x and the last dx are not hidden behind compute. With `graph`, the
    C-ABI forward and backward calls of a step (which allocate nothing and never synchronise)
    are captured once per buffer set into two CUDA graphs and replayed; the copies stay
    outside."""
    import torch
    x_h, dy_h, y_h, dx_h = host
    first = (run.x, run.dy, run.y, run.dx)
    bufs = [first, tuple(torch.empty_like(t) for t in first)]
    graphs = [None, None]
    if graph:
        for b in range(2):
            run.x, run.dy, run.y, run.dx = bufs[b]
            gf, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(gf):
                run.fwd()
            with torch.cuda.graph(gb):
                run.bwd()
            graphs[b] = (gf, gb)
        run.x, run.dy, run.y, run.dx = first
        torch.cuda.synchronize()
    s_in, s_out = torch.cuda.Stream(run.x.device), torch.cuda.Stream(run.x.device)
    ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]  # noqa: E731
    x_ready, dy_ready, fwd_done, comp_done, y_out, dx_out = ev(), ev(), ev(), ev(), ev(), ev()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    s_in.wait_event(t0)
    for i in range(steps):
        b = i & 1
        x, dy, y, dx = bufs[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])  # step i-2 has finished reading x[b], dy[b]
            x.copy_(x_h, non_blocking=True)
            x_ready[b].record(s_in)
            dy.copy_(dy_h, non_blocking=True)
            dy_ready[b].record(s_in)
        stream.wait_event(x_ready[b])
        if i >= 2:
            stream.wait_event(y_out[b])  # step i-2's y[b] has been copied out
        if graphs[b] is not None:
            graphs[b][0].replay()
        else:
            run.x, run.dy, run.y, run.dx = x, dy, y, dx
            run.fwd(stream)
        fwd_done[b].record(stream)
        stream.wait_event(dy_ready[b])
        if i >= 2:
            stream.wait_event(dx_out[b])  # step i-2's dx[b] has been copied out
        if graphs[b] is not None:
            graphs[b][1].replay()
        else:
            run.bwd(stream)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fwd_done[b])
            y_h.copy_(y, non_blocking=True)
            y_out[b].record(s_out)
            s_out.wait_event(comp_done[b])
            dx_h.copy_(dx, non_blocking=True)
            dx_out[b].record(s_out)
    stream.wait_event(dx_out[(steps - 1) & 1])
    t1.record(stream)
    torch.cuda.synchronize()
    run.x, run.dy, run.y, run.dx = first
    return t0.elapsed_time(t1)


def run_mgt(args):
    import torch

    import tensor_transformer_layer_megatron_b200 as mgt
    from mgt_inputs import config_by_name, make_inputs, pack_params, to_sp
    from tensor_transformer_layer_megatron_b200.runner import LayerRun

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = config_by_name(args.config)
    t = make_inputs(cfg)
    packed = pack_params(cfg, t)
    layer = mgt.Layer.from_config(cfg)
    x, dy = t["x"], t["dy"]
    if cfg.sequence_parallel:  # x, dy (and y, dx) in the shard-major sequence-parallel layout
        x, dy = to_sp(cfg, x), to_sp(cfg, dy)
    run = LayerRun(layer, packed, x, dy, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        run.step()
    run.check()
    torch.cuda.synchronize()

    # ---- timed region. With --graph (default) one step (fwd + bwd, 23 kernel launches through
    # the C ABI) is captured once into a CUDA graph and replayed K times; otherwise the C ABI is
    # called eagerly. Per-kernel CUDA events are recorded by the C ABI around every launch of
    # the eager steps (in graph mode: an eager pass of K steps right after the timed replays).
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            run.step()
        graph.replay()
        torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    if not args.graph:
        layer.profile(True)
        layer.profile_read()  # reset totals
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            run.step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    kclocks = ClockSampler(local)  # the eager pass may not run at the timed region's clock
    if args.graph:  # per-kernel breakdown from an eager pass of the same K steps
        layer.profile(True)
        layer.profile_read()
        kclocks.start()
        for _ in range(args.steps):
            run.step()
        torch.cuda.synchronize()
        kclk = kclocks.stop()
    else:
        kclk = clk
    prof = layer.profile_read()
    layer.profile(False)
    run.check()
    del graph
    ms = max_over_ranks(ms, world, dev)
    tokens = cfg.tokens * world
    value, ms_step = job_throughput(cfg.tokens, world, ms, args.steps)
    flops_step = cfg.model_flops() * world
    tflops = flops_step / (ms_step / 1e3) / 1e12

    # ---- end to end through the public API with host buffers (pinned), copies timed
    x_h = run.x.cpu().pin_memory()
    dy_h = run.dy.cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    dx_h = torch.empty_like(x_h).pin_memory()
    barrier()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e2e_steps(run, (x_h, dy_h, y_h, dx_h), args.steps, stream,
                                      graph=args.graph), world, dev)
    barrier()
    # the pipelined copies delivered what the device computed (same inputs every step; the
    # layer's y and dx are deterministic)
    if not (torch.equal(y_h, run.y.cpu()) and torch.equal(dx_h, run.dx.cpu())):
        raise RuntimeError("end-to-end outputs differ from the device-resident step")
    e2e_value, _ = job_throughput(cfg.tokens, world, e2e_ms, args.steps)
    h2d = (x_h.numel() * x_h.element_size() + dy_h.numel() * dy_h.element_size())
    d2h = (y_h.numel() * y_h.element_size() + dx_h.numel() * dx_h.element_size())

    # ---- roofline of the dominant kernel family (the tcgen05 GEMM, all call sites together)
    peaks, peak_src = load_peaks()
    # The contraction peak for the regime the timed region ran in: a region under a second
    # runs at full boost clock (the burst figure, a GEMM timed alone); only a seconds-long
    # region settles under the power cap (the sustained figure).
    regime = "burst" if ms < BURST_REGION_MS else "sustained"
    tc_key = "bf16_tflops" if regime == "burst" else "bf16_tflops_sustained"
    tc_peak = float(peaks[tc_key])
    tc_src = "%s %s (%s regime: timed region %.0f ms %s %.0f ms)" % (
        peak_src, tc_key, regime, ms, "<" if regime == "burst" else ">=", BURST_REGION_MS)
    sm_mhz = kclk["sm_mhz"] if kclk else None  # clock of the pass the kernel times come from
    sites = {k: v for k, v in prof.items() if "/" in k}
    families = {}
    for k, v in prof.items():
        f = families.setdefault(k.split("/")[0], {"launches": 0, "ms": 0.0, "flops": 0.0,
                                                   "bytes": 0.0})
        for q in f:
            f[q] += v[q]
    prof = families
    fam = max(prof.items(), key=lambda kv: kv[1]["ms"]) if prof else (None, None)
    roof = None
    traffic, traffic_src = gemm_traffic(cfg.name)
    if fam[0] is not None:
        name, st = fam
        if st["flops"] > 0:
            achieved = st["flops"] / (st["ms"] / 1e3) / 1e12
            roof = {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1),
                    "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": round(achieved / tc_peak, 4),
                    "peak_source": tc_src,
                    "traffic": traffic, "traffic_source": traffic_src,
                    "launches": st["launches"], "avg_launch_ms": round(st["ms"] / st["launches"], 4),
                    "share_of_step": round(st["ms"] / ms, 4)}
        else:
            achieved = st["bytes"] / (st["ms"] / 1e3) / 1e9
            roof = {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None}
    # every family against its own roofline: contractions against the bf16 peak of the
    # regime (model FLOPs), memory-bound kernels against the HBM copy bandwidth (algorithmic
    # bytes); kcycles_per_step = ms per step x median SM MHz, comparable across clocks
    kernels = {k: {"launches": v["launches"], "ms_per_step": round(v["ms"] / args.steps, 4),
                   **({"kcycles_per_step": round(v["ms"] / args.steps * sm_mhz, 1)}
                      if sm_mhz else {}),
                   **({"tflops": round(v["flops"] / (v["ms"] / 1e3) / 1e12, 1),
                       "frac_of_bf16_peak": round(v["flops"] / (v["ms"] / 1e3) / 1e12 /
                                                  tc_peak, 4)}
                      if v["flops"] else {}),
                   **({"gbs": round(v["bytes"] / (v["ms"] / 1e3) / 1e9, 1),
                       "frac_of_hbm": round(v["bytes"] / (v["ms"] / 1e3) / 1e9 /
                                            peaks["hbm_gbs"], 4)}
                      if v["bytes"] and not v["flops"] else {})}
               for k, v in prof.items()}
    gemm_sites = {k.split("/")[1]: {"ms_per_step": round(v["ms"] / args.steps, 4),
                                    "tflops": round(v["flops"] / (v["ms"] / 1e3) / 1e12, 1),
                                    "frac_of_bf16_peak": round(v["flops"] / (v["ms"] / 1e3) /
                                                               1e12 / tc_peak, 4)}
                  for k, v in sites.items()}
    per_launch = dict(KERNELS_PER_LAUNCH)
    # the LayerNorm backward is one pass plus a reduce up to 512 16-byte vectors per row
    vec = 8 if cfg.dtype == "bf16" else 4
    per_launch["ln_bwd"] = 2 if cfg.hidden // vec <= 512 else 3
    # head_dim 128: D pre-pass, the single backward kernel and the dQ conversion
    per_launch["attn_bwd"] = 3 if cfg.dtype == "bf16" and cfg.hidden // cfg.heads == 128 else 2
    launches = sum(v["launches"] * per_launch.get(k, 1) for k, v in prof.items())

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, args.cpu_tokens)

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if cfg.dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,1) inputs and N(0,0.02) random-init weights)",
            "tflops": round(tflops, 1),
            "frac_of_nominal_2250": round(tflops / NOMINAL_BF16_TFLOPS, 4),
            "frac_of_measured_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
            "frac_of_measured_burst": round(tflops / peaks["bf16_tflops"], 4),
            "peak_regime": regime,
            "frac_of_measured_regime_peak": round(tflops / tc_peak, 4),
            "config": bench_config(cfg, world),
            "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "what": "every step: x, dy pinned host -> device, fwd+bwd via the C ABI "
                            "(%s), y, dx -> pinned host; copies on two copy streams into "
                            "double-buffered device tensors, overlapping the neighbouring "
                            "steps' compute" % ("CUDA-graph replay of the calls" if args.graph
                                                else "eager calls")},
            "roofline": roof,
            "kernels": kernels,
            "kernels_timing": ("CUDA events around every launch, eager pass of the same K steps "
                               "right after the timed graph replays" if args.graph else
                               "CUDA events around every launch inside the timed region"),
            "kernels_clocks": kclk,
            "timed_region": ("CUDA-graph replay of the step (fwd+bwd through the C ABI)"
                             if args.graph else "eager C-ABI calls"),
            "gemm_sites": gemm_sites,
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_gemm_fp8(args):
    """The FP8 (e4m3) GEMM next to the bf16 one on the h=4096 layer's forward GEMM shapes (fp32
    outputs for both): operands quantised once on the device, then K timed launches of each
    GEMM between CUDA events. Prints one JSON line (not the layer-step benchmark)."""
    import torch

    import tensor_transformer_layer_megatron_b200 as mgt
    dev = torch.device("cuda", 0)
    T, h, f = 2048, 4096, 11008
    shapes = {"qkv_fwd": (T, 3 * h, h), "outproj_fwd": (T, h, h), "fc1_fwd": (T, f, h),
              "fc2_fwd": (T, h, f)}
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev).manual_seed(5)
    res, tot = {}, {"fp8": [0.0, 0.0], "bf16": [0.0, 0.0]}
    clocks = ClockSampler(0)
    clocks.start()
    for name, (M, N, K) in shapes.items():
        a = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        b = (torch.randn(N, K, device=dev, generator=g) * 0.02).to(torch.bfloat16)
        qa = torch.empty(M, K, dtype=torch.uint8, device=dev)
        qb = torch.empty(N, K, dtype=torch.uint8, device=dev)
        sa = torch.zeros(2, device=dev)
        sb = torch.zeros(2, device=dev)
        mgt.fp8_quantize(a, qa, sa)
        mgt.fp8_quantize(b, qb, sb)
        c = torch.empty(M, N, device=dev)
        runs = {"fp8": lambda: mgt.gemm_fp8(qa, qb, sa, sb, c, M, N, K, K, K, N, st),
                "bf16": lambda: mgt.gemm_bf16(a, b, c, M, N, K, 0, 0, K, K, N, st)}
        res[name] = {}
        for kind, fn in runs.items():
            for _ in range(max(args.warmup, 3)):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.steps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            fl = 2.0 * M * N * K
            res[name][kind] = {"us": round(ms * 1e3, 1), "tflops": round(fl / ms / 1e9, 1)}
            tot[kind][0] += fl
            tot[kind][1] += ms
    clk = clocks.stop()
    if int(st.item()) != 0:
        raise RuntimeError("device status %d" % int(st.item()))
    fp8 = tot["fp8"][0] / tot["fp8"][1] / 1e9
    bf16 = tot["bf16"][0] / tot["bf16"][1] / 1e9
    peaks, src = load_peaks()
    # e4m3 peak = the bf16 burst figure (timed alone) x the nominal dense ratio 4.5 / 2.25
    f8_peak = 2.0 * float(peaks["bf16_tflops"])
    peak_src = "%s bf16_tflops (burst) x 2, the nominal e4m3:bf16 dense ratio" % src
    print(json.dumps({
        "metric": "FP8 (e4m3, per-tensor scaled) GEMM TFLOP/s on the h=4096 forward GEMM shapes",
        "value": round(fp8, 1), "unit": "TFLOP/s", "higher_is_better": True,
        "bf16_same_shapes_tflops": round(bf16, 1), "speedup_vs_bf16": round(fp8 / bf16, 3),
        "roofline": {"kernel": "gemm_tc2 (e4m3)", "bound": "tensor", "achieved": round(fp8, 1),
                     "peak": round(f8_peak, 1), "unit": "TFLOP/s",
                     "frac": round(fp8 / f8_peak, 4), "peak_source": peak_src,
                     "traffic": None},
        "steps": args.steps, "warmup": args.warmup, "dtype": "e4m3 x e4m3 -> f32",
        "data": "synthetic", "per_shape": res, "clocks": clk,
        "timing": "CUDA events around K back-to-back launches per shape; operands (<= 230 MB) "
                  "partly L2-resident"}), flush=True)


def run_torch(args):
    """Context comparator: the same layer in eager PyTorch on the GPU (cuBLAS GEMMs through
    F.linear on the full unsharded weights, which is what logical TP on one GPU computes;
    flash scaled_dot_product_attention; F.layer_norm; autograd backward with bf16 weight
    gradients). Same inputs, same K/W, CUDA events on the stream. Not the product path."""
    import torch
    import torch.nn.functional as F

    from mgt_inputs import config_by_name, make_inputs

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = config_by_name(args.config)
    t = make_inputs(cfg)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    h, H, d, b, s = cfg.hidden, cfg.heads, cfg.head_dim, cfg.micro_batch, cfg.seq
    names = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o", "ln2_g", "ln2_b", "w1", "b1",
             "w2", "b2")
    P = {k: t[k].to(dev, dt).requires_grad_(True) for k in names if k in t}
    x = t["x"].to(dev, dt).requires_grad_(True)
    dy = t["dy"].to(dev, dt)
    approx = "tanh" if cfg.gelu_tanh else "none"

    def step():
        for v in P.values():
            v.grad = None
        x.grad = None
        ln1 = F.layer_norm(x, (h,), P["ln1_g"], P["ln1_b"], cfg.ln_eps)
        q, k, v = F.linear(ln1, P["w_qkv"], P.get("b_qkv")).view(b, s, 3, H, d).unbind(2)
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2),
                                           v.transpose(1, 2), is_causal=True)
        h1 = x + F.linear(o.transpose(1, 2).reshape(b, s, h), P["w_o"], P.get("b_o"))
        ln2 = F.layer_norm(h1, (h,), P["ln2_g"], P["ln2_b"], cfg.ln_eps)
        u = F.linear(ln2, P["w1"], P.get("b1"))
        if cfg.swiglu:
            gate, up = u.chunk(2, dim=-1)
            a = F.silu(gate) * up
        else:
            a = F.gelu(u, approximate=approx)
        y = h1 + F.linear(a, P["w2"], P.get("b2"))
        y.backward(dy)
        return y

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    value, ms_step = job_throughput(cfg.tokens, world, ms, args.steps)
    tflops = cfg.model_flops() * world / (ms_step / 1e3) / 1e12
    if rank == 0:
        print(json.dumps({
            "impl": "torch-eager", "metric": METRIC, "value": round(value, 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
            "data": "synthetic (same seeded inputs as the main arm)",
            "tflops": round(tflops, 1),
            "what": "context comparator: eager torch (cuBLAS F.linear on unsharded weights, "
                    "flash SDPA, F.layer_norm, autograd; bf16 weight grads)",
            "config": {"workload": cfg.name, "tokens_per_gpu": cfg.tokens},
            "clocks": clk}), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def bench_config(cfg, world):
    """The `config` object of the JSON line (the same on both arms)."""
    return {"workload": cfg.name, "hidden": cfg.hidden, "heads": cfg.heads,
            "mlp": "swiglu" if cfg.swiglu else ("gelu-tanh" if cfg.gelu_tanh else "gelu"),
            "linear_bias": not cfg.disable_bias_linear,
            "sequence_parallel": bool(cfg.sequence_parallel),
            "ffn": cfg.ffn, "seq_len": cfg.seq, "micro_batch": cfg.micro_batch,
            "tp_size": cfg.tp_size, "tokens_per_gpu": cfg.tokens,
            "global_batch": cfg.micro_batch * world,
            "parallelism": "dp%d (independent replicas), logical tp%d per replica"
                           % (world, cfg.tp_size),
            "l2": "no flush: per-step working set (weights 315 MB bf16 + fp32 grads "
                  "630 MB + activations) exceeds the 126 MB L2"}


def cpu_baseline(cfg, tokens):
    """The fp64 oracle, as it stands, on a bounded sample: one sequence of `tokens` tokens of
    the same layer (weights of the full shape), forward + backward, on this host's cores."""
    import torch

    import oracle
    from mgt_inputs import make_inputs, pack_params, to_sp
    sub = cfg.replace(seq=tokens, micro_batch=1)
    t = make_inputs(sub)
    packed = pack_params(sub, t)
    x, dy = t["x"], t["dy"]
    if sub.sequence_parallel:
        x, dy = to_sp(sub, x), to_sp(sub, dy)
    t0 = time.time()
    _, saved = oracle.layer_fwd(sub, packed, x)
    oracle.layer_bwd(sub, packed, saved, dy)
    dt = time.time() - t0
    cores, blas = host_threads()
    return {"value": round(tokens / dt, 3), "unit": "tokens/s",
            "cores": cores, "blas_threads": blas, "kind": "oracle",
            "sample": "fp64 numpy oracle fwd+bwd of one %d-token sequence of the %s layer "
                      "(full weight shapes), %.1f s; matmuls on %s BLAS threads, elementwise "
                      "steps on one" % (tokens, cfg.name, dt, blas)}


def host_threads():
    """Cores this process may run on (its CPU affinity) and the threads numpy's BLAS uses."""
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max((i["num_threads"] for i in threadpool_info() if i["user_api"] == "blas"),
                   default=None)
    except Exception:  # noqa: BLE001 - no threadpoolctl: unknown
        blas = None
    return cores, blas


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mgt_inputs import config_by_name
    cfg = config_by_name(args.config)
    import torch
    samples = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(cfg, args.cpu_tokens)
        if i >= args.warmup:
            samples.append(r)
    v = sum(s["value"] for s in samples) / len(samples)
    ms_step = cfg.tokens / v * 1e3
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(ms_step, 1), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": bench_config(cfg, world),
           "tokens_per_step_sampled": args.cpu_tokens,
           "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s",
                            "cores": samples[0]["cores"],
                            "blas_threads": samples[0]["blas_threads"], "kind": "oracle",
                            "sample": samples[0]["sample"]},
           "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mgt", choices=["mgt", "reference", "torch"])
    ap.add_argument("--gemm-fp8", action="store_true",
                    help="time the FP8 GEMM against the bf16 one on the forward GEMM shapes")
    ap.add_argument("--config", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-tokens", type=int, default=2048)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="time CUDA-graph replays of the step (default)")
    ap.add_argument("--eager", dest="graph", action="store_false",
                    help="time eager C-ABI calls instead")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gemm_fp8:
        run_gemm_fp8(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.impl == "torch":
        run_torch(args)
    else:
        run_mgt(args)


if __name__ == "__main__":
    main()
