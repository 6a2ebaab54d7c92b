#!/usr/bin/env python
"""Benchmark of libgdn, the gated delta rule on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input:
  * prefill: gdn_prefill over one 262,144-token layer (B=1, 48 v-heads /
    16 q-k heads, Dk=Dv=128, chunk 64, bf16 q/k/v, fp32 g/beta/state,
    zero initial state) -- the headline, in Mtok/s per layer;
  * decode: gdn_decode_step for 256 sequences through 48 layers, each layer
    with its own 768 MiB fp32 state updated in place -- reported as state
    GB/s (bytes read + written) in the "decode" object; the same step with
    the states stored in bfloat16 (gdn_decode_step_bf16_state) is its
    "bf16_state" entry.
Inputs are drawn on the device by the seeded generator and are larger than
L2 (8.7 GB per prefill step, 38.6 GB of decode states), so no flush is needed.
For N > 1 (torchrun) every rank runs the same workload on its own GPU with no
data-path collective (weak scaling); timings are the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the prefill workload (the only other use of oracle/ here).
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill Mtok/s per layer; decode-step state GB/s vs 8 TB/s HBM peak"
PREFILL_WL = "long256k"
DECODE_WL = "decode256"
# per-token algorithmic work of the chunked prefill (Dk = Dv = 128, C = 64,
# Hv = 48, Hqk = 16), Gram matrices shared by the 3 v-heads of a q/k head:
#   flops = Hv (4 C Dv + 2 C Dk + 6 Dk Dv) + Hqk 4 C Dk   = 7,602,176
#   bytes = q,k (2*16*128*2) + v (48*128*2) + o (48*128*2) + g,beta (2*48*4) = 33,152
PREFILL_FLOP_PER_TOKEN = 48 * (4 * 64 * 128 + 2 * 64 * 128 + 6 * 128 * 128) + 16 * 4 * 64 * 128
PREFILL_BYTES_PER_TOKEN = 2 * 16 * 128 * 2 + 48 * 128 * 2 * 2 + 2 * 48 * 4


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--case", default=None,
                   help="profiling mode: run one operation of a named workload (layer4k, "
                        "long256k, varlen32: one gdn_prefill call; decode256: one layer's "
                        "gdn_decode_step; decode256_bf16: the same with a bfloat16 state; "
                        "frontend16k, frontend256k: gdn_short_conv_norm on a 16,384- or "
                        "262,144-token layer; fused16k, fused256k: gdn_prefill_conv, the front "
                        "end fused into the pool prefill, on the same) "
                        "W + K times and print its per-call time; no bench line")
    p.add_argument("--kernel", default="auto", choices=["auto", "pool", "cluster", "single_cta", "recurrent"],
                   help="prefill kernel for --case")
    p.add_argument("--tokens", type=int, default=None,
                   help="token count of a single-sequence prefill --case (a reduced sample, e.g. "
                        "for a DRAM-traffic capture)")
    return p.parse_args()


# ------------------------------------------------------------ distributed --

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            if dist.get_backend() == "nccl":
                dist.barrier(device_ids=[self.local_rank])
            else:
                dist.barrier()

    def max(self, x: float) -> float:
        """Max of a float over ranks (the only collective: timing, not data)."""
        if not self.pg:
            return x
        import torch.distributed as dist
        dev = torch.device("cuda", self.local_rank) if dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def weak_scaling_value(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: every rank processed units_per_rank in the timed region."""
    return units_per_rank * world / seconds_max


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """Samples SM clocks and throttle reasons every 20 ms while the timed
    region runs (NVML reads only; nvidia-smi at 200 ms when NVML is missing)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.nvml = None
        self.lines = []
        self.samples = []  # (sm_mhz, max_mhz, reason bits)
        self.active = False
        self.stopping = False

    def _reader(self):
        for line in self.proc.stdout:
            if self.active:
                self.lines.append(line.strip())

    def _poll(self):
        nv, h = self.nvml
        while not self.stopping:
            if self.active:
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(sm), float(mx), int(rs)))
                except Exception:
                    pass
            time.sleep(0.02)

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nvml = (nv, nv.nvmlDeviceGetHandleByIndex(self._physical_index()))
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._reader, daemon=True).start()
        except OSError:
            self.proc = None

    def _physical_index(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [x for x in vis.split(",") if x.strip()]
        if ids and ids[0].strip().isdigit() and self.gpu_index < len(ids):
            return int(ids[self.gpu_index])
        return self.gpu_index

    def mark(self, on: bool):
        self.active = on

    def stop(self):
        sm, mx, reasons = [], None, set()
        if self.nvml is not None:
            self.stopping = True
            self.thread.join(timeout=2)
            for s_mhz, m_mhz, bits in self.samples:
                sm.append(s_mhz)
                mx = m_mhz
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        reasons.add(name)
            src = "nvml 20 ms"
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in self.lines:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
            src = "nvidia-smi 200 ms"
        else:
            return None
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "sampler": src}


# -------------------------------------------------------------- roofline ---

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def traffic_for(kernel_key, src_file):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "gated_deltanet_04_b200", "csrc", src_file)
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel_key \
                        and parts[1] == sha:
                    return float(parts[2])
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ timing --

def time_launches(fn, K, W, dist, stream, sampler=None):
    """W warm-up calls, then K timed calls bracketed by barrier + synchronize.
    Returns (total ms, list of per-call ms) measured with CUDA events on ``stream``."""
    for _ in range(W):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    if sampler:
        sampler.mark(True)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark(False)
    dist.barrier()
    torch.cuda.synchronize()
    return start.elapsed_time(end), [a.elapsed_time(b) for a, b in evs]


def percentiles(each_ms):
    """p50 / p95 / p99 of per-call device times (ms), nearest-rank."""
    xs = sorted(each_ms)
    if not xs:
        return None
    # rank ceil(q n), 1-based; the epsilon keeps q n = 95.00000000000001 at 95
    pick = lambda q: xs[min(len(xs), max(1, math.ceil(q * len(xs) - 1e-9))) - 1]
    return {"p50": pick(0.50), "p95": pick(0.95), "p99": pick(0.99), "calls": len(xs)}


def run_conditions():
    """Host and device facts the numbers were taken under."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    cond = {"cpu_model": model, "nproc": os.cpu_count(), "torch": torch.__version__}
    if torch.cuda.is_available():
        cond["gpu"] = torch.cuda.get_device_name(0)
        cond["cuda_runtime"] = torch.version.cuda
    return cond


def cpu_baseline_prefill(tokens: int):
    """The fp64 oracle on the host cores, on the first ``tokens`` tokens of the
    prefill workload (all 48 heads).  Returns (Mtok/s, seconds, threads)."""
    import oracle
    from gated_deltanet_04_b200 import inputs
    oracle.build()
    inp = inputs.make_prefill(PREFILL_WL, device="cpu", T=tokens)
    t0 = time.perf_counter()
    oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"])
    dt = time.perf_counter() - t0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return tokens / dt / 1e6, dt, threads


def run_reference(args, dist):
    """Reference arm: the fp64 CPU oracle, timed as it stands, on rank 0 only."""
    if dist.rank != 0:
        return 0
    tokens = 16384
    for _ in range(args.warmup):
        cpu_baseline_prefill(tokens)
    secs = []
    for _ in range(args.steps):
        _, dt, threads = cpu_baseline_prefill(tokens)
        secs.append(dt)
    total = sum(secs)
    value = tokens * args.steps / total / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{PREFILL_WL}: B=1 T=262144 Hv=48 Hqk=16 D=128 chunk=64 "
                               f"(sample: first {tokens} tokens, all 48 heads, per step)"},
        "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {tokens} tokens x 48 heads of the 262,144-token layer"},
        "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_case(args):
    """Profiling mode: W + K calls of one operation on one GPU, per-call device time."""
    import gated_deltanet_04_b200 as gdn
    from gated_deltanet_04_b200 import inputs
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    if args.case == "decode256":
        L = inputs.make_decode_layer(0, device=dev)
        out = torch.empty_like(L["v"])
        fn = lambda: gdn.gdn_decode_step(L["q"], L["k"], L["v"], L["g"], L["beta"], L["state"], o=out)
    elif args.case in ("frontend16k", "frontend256k"):
        inp = (inputs.make_prefill("layer4k", device=dev, T=16384) if args.case == "frontend16k"
               else inputs.make_prefill("long256k", device=dev))
        gen = torch.Generator(device=dev).manual_seed(1200)
        Hqk_, Hv_ = inp["q"].shape[1], inp["v"].shape[1]
        fw = [0.5 * torch.randn(H * 128, 4, generator=gen, device=dev) for H in (Hqk_, Hqk_, Hv_)]
        fo = [torch.empty_like(inp[key]) for key in ("q", "k", "v")]
        lib = gdn.library()
        Tn = inp["q"].shape[0]
        fn = lambda: lib.gdn_short_conv_norm(inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(),
                                             0, fw[0].data_ptr(), fw[1].data_ptr(), fw[2].data_ptr(),
                                             None, None, None, 1, Tn, Hqk_, Hv_, 128, 128,
                                             fo[0].data_ptr(), fo[1].data_ptr(), fo[2].data_ptr(),
                                             None, stream.cuda_stream)
    elif args.case in ("fused16k", "fused256k"):
        inp = (inputs.make_prefill("layer4k", device=dev, T=16384) if args.case == "fused16k"
               else inputs.make_prefill("long256k", device=dev))
        gen = torch.Generator(device=dev).manual_seed(1200)
        Hqk_, Hv_ = inp["q"].shape[1], inp["v"].shape[1]
        fw = [0.5 * torch.randn(H * 128, 4, generator=gen, device=dev) for H in (Hqk_, Hqk_, Hv_)]
        o = torch.empty_like(inp["v"])
        sT = torch.empty((1, Hv_, 128, 128), dtype=torch.float32, device=dev)
        fst = torch.empty((1, 3, (2 * Hqk_ + Hv_) * 128), dtype=torch.float32, device=dev)
        ws = torch.empty(gdn.gdn_prefill_conv_workspace_bytes(1, inp["T"], Hqk_, Hv_, 128, 128),
                         dtype=torch.uint8, device=dev)
        fn = lambda: gdn.gdn_prefill_conv(inp["q"], inp["k"], inp["v"], fw[0], fw[1], fw[2], inp["g"],
                                          inp["beta"], conv_state_out=fst, o=o, final_state=sT,
                                          workspace=ws)
    elif args.case == "decode256_bf16":
        L = inputs.make_decode_layer(0, device=dev)
        out = torch.empty_like(L["v"])
        sb = L["state"].to(torch.bfloat16)
        fn = lambda: gdn.gdn_decode_step_bf16_state(L["q"], L["k"], L["v"], L["g"], L["beta"], sb,
                                                    o=out)
    else:
        inp = inputs.make_prefill(args.case, device=dev, T=args.tokens)
        o = torch.empty_like(inp["v"])
        N = inp["N"]
        sT = torch.empty((N, inp["wl"].Hv, 128, 128), dtype=torch.float32, device=dev)
        kern = args.kernel
        ws = torch.empty(max(1, gdn.gdn_prefill_workspace_bytes(N, inp["T"], 16, 48, 128, 128, 64,
                                                                kern)), dtype=torch.uint8, device=dev)
        fn = lambda: gdn.gdn_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                     inp["s0"], inp["cu_seqlens"], chunk=inp["wl"].chunk,
                                     o=o, final_state=sT, workspace=ws, kernel=kern)
    total, each = time_launches(fn, args.steps, args.warmup, Dist(), stream)
    print(json.dumps({"case": args.case, "kernel": args.kernel, "calls": args.steps, "ms_per_call": total / args.steps,
                      "ms_min": min(each), "ms_max": max(each)}), flush=True)
    return 0


def main():
    args = parse()
    if args.case:
        return run_case(args)
    dist = Dist()
    if args.impl == "reference":
        dist.init("gloo")
        rc = run_reference(args, dist)
        dist.close()
        return rc

    import gated_deltanet_04_b200 as gdn
    from gated_deltanet_04_b200 import inputs

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(dist.local_rank)
    dist.init("nccl")
    gdn.library()  # fails loudly when libgdn.so is missing
    dev = torch.device("cuda", dist.local_rank)
    stream = torch.cuda.current_stream()
    K, W = args.steps, max(3, args.warmup)
    peaks = measured_peaks()
    sampler = ClockSampler(dist.local_rank)
    sampler.start()

    # ---------------------------------------------------------- prefill --
    inp = inputs.make_prefill(PREFILL_WL, device=dev)
    T = inp["T"]
    o = torch.empty_like(inp["v"])
    sT = torch.empty((1, 48, 128, 128), dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, gdn.gdn_prefill_workspace_bytes(1, T, 16, 48, 128, 128, 64)),
                     dtype=torch.uint8, device=dev)

    def prefill():
        gdn.gdn_prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None,
                        chunk=64, o=o, final_state=sT, workspace=ws)

    p_total, p_each = time_launches(prefill, K, W, dist, stream, sampler)
    p_ms = dist.max(p_total / K)
    p_launch_ms = dist.max(sum(p_each) / K)
    del o, sT

    # ------------------------------------------- the other prefill workloads --
    # the 4096-token layer (pool kernel) and the 32-sequence varlen batch (1,536
    # units: the single-CTA kernel), each in Mtok/s with per-call percentiles
    others = {}
    for name, calls in (("layer4k", max(K, 50)), ("varlen32", K)):
        winp = inputs.make_prefill(name, device=dev)
        wo = torch.empty_like(winp["v"])
        wsT = torch.empty((winp["N"], 48, 128, 128), dtype=torch.float32, device=dev)
        wws = torch.empty(max(1, gdn.gdn_prefill_workspace_bytes(winp["N"], winp["T"], 16, 48, 128,
                                                                 128, 64)),
                          dtype=torch.uint8, device=dev)

        def wcall(winp=winp, wo=wo, wsT=wsT, wws=wws):
            gdn.gdn_prefill(winp["q"], winp["k"], winp["v"], winp["g"], winp["beta"], winp["s0"],
                            winp["cu_seqlens"], chunk=64, o=wo, final_state=wsT, workspace=wws)

        w_total, w_each = time_launches(wcall, calls, W, dist, stream, sampler)
        w_ms = dist.max(w_total / calls)
        others[name] = {"value": weak_scaling_value(winp["T"], w_ms / 1e3, dist.world) / 1e6,
                        "unit": "Mtok/s", "ms_per_call": w_ms, "tokens": winp["T"],
                        "units": winp["N"] * 48,
                        "kernel": "pool" if winp["N"] * 48 <= 64 else "single_cta",
                        "percentiles_ms": percentiles(w_each)}
        del winp, wo, wsT, wws
    o = torch.empty_like(inp["v"])
    sT = torch.empty((1, 48, 128, 128), dtype=torch.float32, device=dev)

    # ------------------------------------------------------- front end --
    # the kernel-4 short convolution + q/k norm over the same layer's q, k, v
    # channels (the prefill inputs serve as its raw inputs), with a conv state out
    gen = torch.Generator(device=dev).manual_seed(1200)
    Hqk_, Hv_ = inp["q"].shape[1], inp["v"].shape[1]
    fw = [0.5 * torch.randn(H * 128, 4, generator=gen, device=dev) for H in (Hqk_, Hqk_, Hv_)]
    fq, fk, fv = torch.empty_like(inp["q"]), torch.empty_like(inp["k"]), torch.empty_like(inp["v"])
    fst = torch.empty((1, 3, (2 * Hqk_ + Hv_) * 128), dtype=torch.float32, device=dev)
    lib = gdn.library()

    def front_end():
        lib.gdn_short_conv_norm(inp["q"].data_ptr(), inp["k"].data_ptr(), inp["v"].data_ptr(), 0,
                                fw[0].data_ptr(), fw[1].data_ptr(), fw[2].data_ptr(), None,
                                fst.data_ptr(), None, 1, T, Hqk_, Hv_, 128, 128, fq.data_ptr(),
                                fk.data_ptr(), fv.data_ptr(), None, stream.cuda_stream)

    f_total, f_each = time_launches(front_end, K, W, dist, stream, sampler)
    f_ms = dist.max(f_total / K)
    f_bytes = 2 * sum(t.numel() * t.element_size() for t in (fq, fk, fv)) + \
        sum(w.numel() * 4 for w in fw) + fst.numel() * 4
    del fq, fk, fv

    # the same front end fused into the pool prefill (gdn_prefill_conv): the
    # layer's raw channels in, o, final state and conv state out
    cws = torch.empty(gdn.gdn_prefill_conv_workspace_bytes(1, T, Hqk_, Hv_, 128, 128),
                      dtype=torch.uint8, device=dev)

    def fused():
        gdn.gdn_prefill_conv(inp["q"], inp["k"], inp["v"], fw[0], fw[1], fw[2], inp["g"],
                             inp["beta"], conv_state_out=fst, o=o, final_state=sT, workspace=cws)

    u_total, u_each = time_launches(fused, K, W, dist, stream, sampler)
    u_ms = dist.max(u_total / K)
    del fw, fst, cws

    # ----------------------------------------------------------- decode --
    dwl = inputs.WORKLOADS[DECODE_WL]
    layers = [inputs.make_decode_layer(l, device=dev) for l in range(dwl.layers)]
    d_outs = [torch.empty_like(L["v"]) for L in layers]

    def decode_step():
        for L, out in zip(layers, d_outs):
            gdn.gdn_decode_step(L["q"], L["k"], L["v"], L["g"], L["beta"], L["state"], o=out)

    d_total, d_each = time_launches(decode_step, K, W, dist, stream, sampler)
    d_ms = dist.max(d_total / K)
    state_bytes_layer = dwl.N * dwl.Hv * dwl.Dv * dwl.Dk * 4 * 2
    io_bytes_layer = dwl.N * (2 * dwl.Hqk * dwl.Dk * 2 + 2 * dwl.Hv * dwl.Dv * 2 + 2 * dwl.Hv * 4)
    d_state_gbs = weak_scaling_value(state_bytes_layer * dwl.layers, d_ms / 1e3, dist.world) / 1e9
    # per-launch timing of the decode kernel (one layer), for its roofline
    L0, out0 = layers[0], d_outs[0]
    d1_total, _ = time_launches(
        lambda: gdn.gdn_decode_step(L0["q"], L0["k"], L0["v"], L0["g"], L0["beta"], L0["state"],
                                    o=out0), K, W, dist, stream)
    d1_ms = dist.max(d1_total / K)
    # the same step with each layer's state stored in bfloat16 (half the bytes)
    b_states = [L["state"].to(torch.bfloat16) for L in layers]

    def decode_step_bf16():
        for L, st, out in zip(layers, b_states, d_outs):
            gdn.gdn_decode_step_bf16_state(L["q"], L["k"], L["v"], L["g"], L["beta"], st, o=out)

    b_total, b_each = time_launches(decode_step_bf16, K, W, dist, stream, sampler)
    b_ms = dist.max(b_total / K)
    b_state_gbs = weak_scaling_value(state_bytes_layer // 2 * dwl.layers, b_ms / 1e3,
                                     dist.world) / 1e9
    del layers, d_outs, b_states
    torch.cuda.empty_cache()
    clocks = sampler.stop()

    # -------------------------------------------------------------- e2e --
    e2e = None
    if not args.no_e2e:
        # gdn_prefill_host: pinned host inputs and outputs, the layer streamed
        # through the device in 16,384-token segments that carry the state, the
        # copies in and out overlapping the kernels
        host = {key: inp[key].cpu().pin_memory() for key in ("q", "k", "v", "g", "beta")}
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        s_host = torch.empty(sT.shape[1:], dtype=sT.dtype).pin_memory()
        del o, sT, ws, inp
        torch.cuda.empty_cache()
        scratch = torch.empty(gdn.gdn_prefill_host_scratch_bytes(T, 16, 48, 128, 128, 64),
                              dtype=torch.uint8, device=dev)

        def e2e_step():
            gdn.gdn_prefill_host(host["q"], host["k"], host["v"], host["g"], host["beta"], None,
                                 o=o_host, final_state=s_host, chunk=64, scratch=scratch,
                                 device=dev)

        e_total, e_each = time_launches(e2e_step, K, W, dist, stream)
        e_ms = dist.max(e_total / K)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_host.numel() * o_host.element_size() + s_host.numel() * s_host.element_size()
        e2e = {"value": weak_scaling_value(T, e_ms / 1e3, dist.world) / 1e6, "unit": "Mtok/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "percentiles_ms": percentiles(e_each)}

    # --------------------------------------------------------- roofline --
    # Dk = Dv = 128, bf16, chunk 64, 48 units: the library's default is the pool kernel
    flops = PREFILL_FLOP_PER_TOKEN * T
    achieved_tf = flops / (p_launch_ms / 1e3) / 1e12
    achieved_gbs = PREFILL_BYTES_PER_TOKEN * T / (p_launch_ms / 1e3) / 1e9
    roofline = {"bound": "tensor", "achieved": achieved_tf, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved_tf / peaks["bf16_tflops"],
                "traffic": traffic_for("gdn_prefill_pool", "prefill_chain.cu"),
                "peak_source": f"{peaks['source']} bf16 burst",
                "kernel": "gdn_prefill_pool_kernel",
                "algorithmic_flop_per_launch": flops,
                "hbm": {"achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved_gbs / peaks["hbm_gbs"],
                        "algorithmic_bytes_per_launch": PREFILL_BYTES_PER_TOKEN * T}}
    d_gbs_launch = (state_bytes_layer + io_bytes_layer) / (d1_ms / 1e3) / 1e9
    decode = {"value": d_state_gbs, "unit": "GB/s", "ms_per_step": d_ms,
              "percentiles_ms": percentiles(d_each),
              "layers_per_step": dwl.layers, "sequences": dwl.N,
              "roofline": {"bound": "hbm", "achieved": d_gbs_launch, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": d_gbs_launch / peaks["hbm_gbs"],
                           "traffic": traffic_for("gdn_decode", "decode.cu"),
                           "peak_source": f"{peaks['source']} copy",
                           "kernel": "gdn_decode_staged_kernel",
                           "algorithmic_bytes_per_launch": state_bytes_layer + io_bytes_layer},
              "frac_of_8TBps": d_state_gbs / dist.world / 8000.0,
              "bf16_state": {"value": b_state_gbs, "unit": "GB/s", "ms_per_step": b_ms,
                             "percentiles_ms": percentiles(b_each),
                             "note": "same 48-layer step with the state stored in bfloat16 "
                                     "(gdn_decode_step_bf16_state); GB/s of bf16 state bytes",
                             "frac_of_measured_copy": b_state_gbs / dist.world / peaks["hbm_gbs"],
                             "frac_of_8TBps": b_state_gbs / dist.world / 8000.0}}

    front = {"value": weak_scaling_value(T, f_ms / 1e3, dist.world) / 1e6, "unit": "Mtok/s",
             "ms_per_step": f_ms, "percentiles_ms": percentiles(f_each),
             "note": "gdn_short_conv_norm (kernel-4 causal conv on q, k, v channels, q/k L2 "
                     "norm) over the same 262,144-token layer",
             "hbm": {"achieved": f_bytes / (f_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": f_bytes / (f_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "algorithmic_bytes_per_launch": f_bytes}}

    fused_line = {"value": weak_scaling_value(T, u_ms / 1e3, dist.world) / 1e6, "unit": "Mtok/s",
                  "ms_per_step": u_ms, "percentiles_ms": percentiles(u_each),
                  "separate_calls_ms": f_ms + p_ms,
                  "note": "gdn_prefill_conv: the front end above fused into the pool prefill "
                          "(filter rearrangement, pool kernel, conv-state kernel) over the "
                          "same 262,144-token layer; separate_calls_ms = front end + prefill"}

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        tokens = 65536
        val, dt, threads = cpu_baseline_prefill(tokens)
        cpu = {"value": val, "unit": "Mtok/s", "cores": threads, "kind": "oracle",
               "sample": f"first {tokens} tokens x 48 heads of the 262,144-token layer, "
                         f"{dt:.1f} s"}

    line = {
        "metric": METRIC,
        "value": weak_scaling_value(T, p_ms / 1e3, dist.world) / 1e6,
        "unit": "Mtok/s",
        "n_gpus": dist.world, "steps": K, "warmup": W, "ms_per_step": p_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{PREFILL_WL}: prefill B=1 T=262144 Hv=48 Hqk=16 Dk=Dv=128 "
                               f"chunk=64 bf16 q/k/v, fp32 g/beta/state; plus {DECODE_WL}: "
                               "decode N=256 x 48 layers (see 'decode')",
                   "l2": "inputs larger than L2 (8.7 GB per prefill, 38.6 GB decode states)",
                   "parallelism": f"replica x{dist.world} (no data-path collective)"},
        "percentiles_ms": percentiles(p_each),
        "roofline": roofline,
        "prefill_workloads": others,
        "decode": decode,
        "front_end": front,
        "front_end_fused": fused_line,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": K * (1 + 2 + 3 + dwl.layers + 1 + dwl.layers)
                        + K * (0 if args.no_e2e else -(-T // 16384)) + max(K, 50) + K,
        "clocks": clocks,
        "run_conditions": run_conditions(),
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
