"""Benchmark of the sparse top-k MoE layer forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

Workload: the Mixtral-shaped layer (T=4096 tokens, H=4096, E=8 experts, top-2, F=14336, GELU FFN
with biases, dropless; bf16 storage, fp32 accumulation), synthetic seeded inputs.  A step is one
whole forward pass (router, permutation, both grouped GEMMs with the fused combine) through the
C-ABI call moe_forward; inputs are resident in HBM when the timed region starts.  The expert
weights (1.88 GB) stream through L2 every step, so the inputs are larger than L2 and no flush is
needed.  ``e2e`` times moe_forward_host: per step it copies x from pinned host memory to the device
and out back to pinned host memory; three buffer sets on three streams let one step's copies overlap
the other steps' kernels (the one-stream figure is reported beside it).  With N GPUs (torchrun), every rank runs its own replica on its
own batch (no data-path collective; the layer shards by tokens), timing is the max over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded token sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer fwd tokens/sec (Mixtral shape, 1 B200); grouped-GEMM % of BF16 peak"


def workload_config(cfg: synth.LayerConfig) -> str:
    cf = "dropless" if math.isinf(cfg.CF) else f"CF={cfg.CF}"
    ffn = f"{cfg.act.upper()} FFN " + ("with biases" if cfg.bias else "without biases")
    route = "" if cfg.routing == "token_choice" else f"{cfg.routing.replace('_', '-')} routing, "
    return (f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} k={cfg.k} F={cfg.F} {cf}, {route}{ffn}, "
            f"{cfg.dtype} storage / fp32 accumulate")


def alg_flops(cfg: synth.LayerConfig, kept: int) -> float:
    """4*H*F per kept assignment (two GEMMs) + 2*T*H*E for the gate."""
    return 4.0 * cfg.H * cfg.F * kept + 2.0 * cfg.T * cfg.H * cfg.E


def alg_bytes(cfg: synth.LayerConfig, touched_experts: int) -> float:
    es = 2 if cfg.dtype == "bf16" else 4
    w = touched_experts * (2 * cfg.H * cfg.F + (cfg.F + cfg.H if cfg.bias else 0)) * es
    return w + cfg.T * cfg.H * es + cfg.T * cfg.H * 4 + cfg.H * cfg.E * es


def ffn_alg_bytes(cfg: synth.LayerConfig, kept: int, touched_experts: int) -> float:
    """Algorithmic DRAM bytes of one moe_expert_ffn call: the touched experts' W1, W2 (and biases)
    once, x_perm read, h written and read back (storage dtype), out read and written (fp32)."""
    es = 2 if cfg.dtype == "bf16" else 4
    w = touched_experts * (2 * cfg.H * cfg.F + (cfg.F + cfg.H if cfg.bias else 0)) * es
    return w + kept * cfg.H * es + 2 * kept * cfg.F * es + 2 * cfg.T * cfg.H * 4


# dense bf16 tcgen05 rate of one SM per clock (the nominal 2.25 PFLOP/s of 148 SMs at 1.855 GHz)
TC_FLOP_PER_CLK_SM = 8192


# Back-to-back grouped GEMMs at the Mixtral shape ran at the burst clock for about the first 75 ms;
# then the 1 kW power cap lowered the SM clock (a probe of 1000 calls with a clock reading every 10 ms).
CAP_ONSET_S = 0.075


def ffn_roofline(cfg: synth.LayerConfig, kept: int, touched_experts: int, ms_ffn: float, peaks: dict,
                 clocks: dict | None = None, sms: int = 148, loop_s: float | None = None) -> dict:
    """Roofline object of the dominant kernel pair (one moe_expert_ffn call): tensor-bound when its
    FLOPs take longer at the bf16 peak than its algorithmic bytes at the copy bandwidth, else
    HBM-bound (weight streaming: decode, the Switch shape).  The calls are timed on their own in a loop
    of loop_s seconds: shorter than the power cap's onset, the peak is the measured burst bf16 figure;
    longer, the measured sustained (power-capped) one.  Both fractions are kept.  With the clock record
    of the same timing loop, the tensor rate per SM-cycle (time x median SM MHz) is given against the
    nominal 8192 FLOP/clk/SM."""
    flops = 4.0 * cfg.H * cfg.F * kept
    nbytes = ffn_alg_bytes(cfg, kept, touched_experts)
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    sec = ms_ffn / 1000.0
    if t_tensor >= t_hbm:
        a = flops / sec / 1e12
        capped = loop_s is not None and loop_s >= CAP_ONSET_S
        pk = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
        regime = (f"sustained (a {loop_s:.2f} s loop, past the power cap's onset)" if capped else
                  "burst (kernel timed alone, before the power cap engages)")
        r = {"bound": "tensor", "achieved": a, "peak": pk, "unit": "TFLOP/s", "frac": a / pk,
             "peak_source": f"{peaks['source']} bf16 {regime}",
             "frac_of_burst": a / peaks["bf16_tflops"],
             "frac_of_sustained": a / peaks["bf16_tflops_sustained"]}
    else:
        a, pk = nbytes / sec / 1e9, peaks["hbm_gbs"]
        r = {"bound": "hbm", "achieved": a, "peak": pk, "unit": "GB/s", "frac": a / pk,
             "peak_source": f"{peaks['source']} HBM copy"}
    r["algorithmic"] = {"flops": flops, "bytes": nbytes}
    mhz = (clocks or {}).get("sm_mhz")
    if mhz:
        per_clk = flops / (sec * mhz * 1e6 * sms)
        r["tensor_flop_per_sm_clk"] = {"value": per_clk, "of_nominal": per_clk / TC_FLOP_PER_CLK_SM,
                                       "sm_mhz_median": mhz, "sms": sms}
    return r


def sustained_roofline(cfg: synth.LayerConfig, kept: int, ms: float, peaks: dict, clocks: dict | None,
                       sms: int = 148) -> dict:
    """The same call timed in a loop of about 0.3 s, long enough for the power cap to set the clock: its
    rate against the measured sustained (power-capped) bf16 peak, and per SM-cycle at that clock."""
    flops = 4.0 * cfg.H * cfg.F * kept
    a = flops / (ms / 1000.0) / 1e12
    r = {"ms": ms, "achieved": a, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
         "frac": a / peaks["bf16_tflops_sustained"], "clocks": clocks}
    mhz = (clocks or {}).get("sm_mhz")
    if mhz:
        per_clk = flops / (ms / 1000.0 * mhz * 1e6 * sms)
        r["tensor_flop_per_sm_clk"] = {"value": per_clk, "of_nominal": per_clk / TC_FLOP_PER_CLK_SM}
    return r


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """SM clock, power and throttle reasons sampled while running: NVML polled every `interval_ms`
    (fine enough to resolve a loop of a few tens of milliseconds), else nvidia-smi every 50 ms.  Only
    readings are taken; no setting of the GPU is touched."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_id: str | None, interval_ms: float = 2.0):
        self.gpu_id = gpu_id
        self.interval = interval_ms / 1000.0
        self.proc = None
        self.thread = None
        self.stop_flag = False
        self.samples = []  # (time, sm_mhz, sm_max_mhz, power_w, reasons bitmask, power_limit_w, temp_c)
        self.window = None  # host-time bounds of the measured region (mark), else every sample
        self.lines = []
        self.source = None

    def start(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id) if self.gpu_id
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            self._nvml, self._h = pynvml, h
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.plimit = pynvml.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        except Exception:
            self._nvml = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
        if self.gpu_id:
            cmd.insert(1, f"--id={self.gpu_id}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi"
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,power.limit,temperature.gpu")

    def mark(self, t0: float, t1: float):
        """Keep only the samples taken between host times t0 and t1 (the region being measured)."""
        self.window = (t0, t1)

    def _poll_nvml(self):
        nv, h = self._nvml, self._h
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                tc = nv.nvmlDeviceGetTemperature(h, nv.NVML_TEMPERATURE_GPU)
                self.samples.append((time.time(), float(sm), float(self.smax), pw, rs, self.plimit, float(tc)))
            except Exception:
                pass
            time.sleep(self.interval)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampler unavailable"]}
        self.stop_flag = True
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, power, reasons, plimit, temp = [], [], [], set(), [], []
        if self.source == "nvml":
            rows = self.samples
            if self.window is not None:
                inside = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
                rows = inside or rows
            for _, s_, mx, pw, rs, pl, tc in rows:
                sm.append(s_)
                smax.append(mx)
                power.append(pw)
                plimit.append(pl)
                temp.append(tc)
                for n, bit in self.REASONS:
                    if rs & bit:
                        reasons.add(n)
        else:
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for ln in self.lines:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                    power.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
                try:
                    plimit.append(float(parts[8]))
                    temp.append(float(parts[9]))
                except (ValueError, IndexError):
                    pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        if self.source == "nvml" and self.window is not None:
            loaded = sm  # already the samples of the measured region
        else:
            thr = max(power) * 0.5 if power else 0
            loaded = [s for s, p in zip(sm, power) if p >= thr] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "samples_loaded": len(loaded), "source": self.source,
                "power_w_max": max(power) if power else None,
                "power_w_median": statistics.median(power) if power else None,
                "power_limit_w": max(plimit) if plimit else None, "temp_c_max": max(temp) if temp else None}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def replica_inputs(cfg: synth.LayerConfig, rank: int, with_weights: bool = True) -> synth.LayerInputs:
    """Inputs of one data-parallel replica: the shared layer weights and this rank's own batch."""
    inp = synth.make_inputs(cfg, with_weights=with_weights)
    if rank > 0:
        inp.x = synth.x_batch(cfg, rank)
    return inp


def max_over_ranks(v: float, world: int, device=None) -> float:
    """Slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, tokens_per_rank: int, steps: int, ms_total_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_total_max / 1000.0)


# ------------------------------------------------------------------------------------------------
def oracle_layer(cfg: synth.LayerConfig, inp: synth.LayerInputs, lo: int, n: int):
    """The fp64 oracle's whole layer on tokens [lo, lo+n) taken as one batch, under the workload's
    routing rule."""
    import oracle

    fwd = oracle.forward_ec if cfg.routing == "expert_choice" else oracle.forward
    return fwd(inp.x[lo:lo + n], inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype,
               act=cfg.act)


def cpu_oracle_rate(cfg: synth.LayerConfig, inp: synth.LayerInputs, budget_s: float, max_tokens: int = 4096):
    """Tokens/s of the fp64 oracle (routing + dispatch + FFN + combine) on a leading token sample,
    growing the sample until one run lasts at least budget_s / 3."""
    import oracle

    oracle.build()
    threads = oracle.max_threads()
    n = 2
    best = None
    spent = 0.0
    while True:
        t0 = time.perf_counter()
        oracle_layer(cfg, inp, 0, n)
        dt = time.perf_counter() - t0
        spent += dt
        best = (n, dt)
        if dt >= budget_s / 3 or n >= min(max_tokens, cfg.T) or spent + 2.2 * dt > budget_s:
            break
        n = min(n * 2, cfg.T)  # the sample never runs past the batch
    n, dt = best
    # one core on a small leading sample, for the single-core figure (extrapolated to the whole batch)
    n1 = max(1, min(n, 8))
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle_layer(cfg, inp, 0, n1)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(threads)
    return {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"first {n} tokens of the {cfg.name} workload as one layer call (routing, dispatch, "
                      f"expert FFN, combine in fp64), {dt:.2f} s",
            "full_batch_estimate_s": cfg.T * dt / n,
            "single_core": {"value": n1 / dt1, "unit": "tokens/s", "cores": 1, "extrapolated": True,
                            "sample": f"first {n1} tokens on one thread, {dt1:.2f} s; the whole {cfg.T}-token "
                                      f"batch would take about {cfg.T * dt1 / n1:.0f} s"}}


def run_reference(args, cfg):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle

    inp = synth.make_inputs(cfg)
    oracle.build()
    threads = oracle.max_threads()
    # calibrate tokens per step so the whole run stays within about two minutes
    t0 = time.perf_counter()
    oracle_layer(cfg, inp, 0, 1)
    t1 = time.perf_counter() - t0
    per_step = 120.0 / max(1, args.steps + args.warmup)
    S = int(max(1, min(cfg.T, per_step / max(t1, 1e-6))))
    for _ in range(args.warmup):
        oracle_layer(cfg, inp, 0, S)
    t0 = time.perf_counter()
    for i in range(args.steps):
        lo = (i * S) % max(1, cfg.T - S + 1)
        oracle_layer(cfg, inp, lo, S)
    dt = time.perf_counter() - t0
    value = S * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_config(cfg), "global_batch": S, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{S} tokens per step of the {cfg.name} workload (fp64 oracle, OpenMP)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
def captured_traffic(workload: str):
    """DRAM bytes of one moe_expert_ffn call on `workload` from the committed ncu capture, or None
    when there is none or a kernel source has changed since it was taken (sha256 mismatch)."""
    import hashlib

    try:
        entry = json.load(open(os.path.join(ROOT, "profiles", "traffic.json"))).get(workload)
        if not entry:
            return None
        for rel, digest in entry["sources_sha256"].items():
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        return entry["grouped_gemm_bytes_per_launch"]
    except (OSError, ValueError, KeyError, TypeError):
        return None


def _upload(arr, dtype):
    import torch

    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def run_ours_impl(args, cfg):
    import torch
    import torch.distributed as dist

    import sparse_mixture_experts_23_b200 as moe
    from sparse_mixture_experts_23_b200 import build as moe_build

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=torch.device("cuda", local))
        if rank == 0:
            moe_build.build()
        dist.barrier()
    else:
        moe_build.build()
    moe.load_library()

    inp = replica_inputs(cfg, rank)
    dev = {n: _upload(a, cfg.dtype) for n, a in inp.arrays().items()}
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.k, cfg.F, cfg.CF, cfg.dtype, cfg.act, cfg.routing)
    buf = moe.MoEBuffers(shape, dev)
    stream = torch.cuda.current_stream()
    peaks = load_peaks()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid if rank == 0 else None)

    def sync_all():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        buf.forward()
    if rank == 0:
        sampler.start()
        time.sleep(0.1)  # let the sampler take its first readings
    # ---------------- timed region: K whole forward passes -----------------------------------
    sync_all()
    t_host0 = time.time()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        buf.forward()
    ev1.record(stream)
    sync_all()
    if rank == 0:
        sampler.mark(t_host0, time.time())
    clocks = sampler.stop() if rank == 0 else None
    launches_per_step = moe.moe_last_launch_count()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world, "cuda")
    ms_step = ms_total / args.steps
    value = aggregate_rate(world, cfg.T, args.steps, ms_total)

    # ---------------- e2e: host buffers through moe_forward_host ----------------------------
    # Every step copies its x from pinned host memory, runs the layer and copies out back to pinned
    # host memory, all inside the timed region.  "serial": one stream, so each step's copies wait for
    # the previous step's kernels.  "pipelined" (the reported value): three device buffer sets on
    # three streams, steps rotating between them, so the host copies of some steps run on the copy
    # engines while another step's kernels run -- what a caller streaming batches through the layer
    # does (calls on distinct workspaces may run concurrently on distinct streams).  Both run right
    # after the device-timed region and an idle pause, before the power-capped GEMM loops below.
    es = 2 if cfg.dtype == "bf16" else 4
    x_np = np.ascontiguousarray(inp.x).view(np.int16 if es == 2 else np.float32)

    def host_pair():
        xh = torch.from_numpy(x_np.copy())
        if es == 2:
            xh = xh.view(torch.bfloat16)
        return xh.pin_memory(), torch.empty((cfg.T, cfg.H), dtype=torch.float32).pin_memory()

    NBUF = 3  # buffer sets for the pipelined figure (triple buffering)
    hosts = [host_pair() for _ in range(NBUF)]
    for _ in range(2):
        buf.forward_host(*hosts[0])
    sync_all()
    time.sleep(0.5)  # rested clocks, as for the device-timed region
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        buf.forward_host(*hosts[0])
    e1.record(stream)
    sync_all()
    ms_e2e_serial = max_over_ranks(e0.elapsed_time(e1), world, "cuda")

    extra = []
    for _ in range(NBUF - 1):
        inputs_j = dict(buf.inputs)
        inputs_j["x"] = torch.empty_like(buf.inputs["x"])  # moe_forward_host writes the step's x here
        extra.append(moe.MoEBuffers(shape, inputs_j))
    bufs = [buf] + extra
    streams = [torch.cuda.Stream() for _ in range(NBUF)]

    def pipelined(n):
        # step i runs on buffer set i % NBUF and its own stream: the copies of one step overlap the
        # kernels of the others, and a set's next input copy waits only for its own previous output
        for i in range(n):
            with torch.cuda.stream(streams[i % NBUF]):
                bufs[i % NBUF].forward_host(*hosts[i % NBUF])

    for s_ in streams:
        s_.wait_stream(torch.cuda.current_stream())
    pipelined(2 * NBUF)
    sync_all()
    time.sleep(0.5)
    e0.record(stream)
    for s_ in streams:
        s_.wait_event(e0)
    pipelined(args.steps)
    for s_ in streams:
        stream.wait_stream(s_)
    e1.record(stream)
    sync_all()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    e2e_value = aggregate_rate(world, cfg.T, args.steps, ms_e2e)
    e2e_serial = aggregate_rate(world, cfg.T, args.steps, ms_e2e_serial)
    out_diff = max(float((hosts[0][1] - h[1]).abs().max()) for h in hosts[1:])  # every set ran the same x
    e2e_status = max(b.device_status() for b in bufs)
    del extra, bufs

    # ---------------- per-kernel timing (same stream, CUDA events, inputs > L2) ---------------
    reps = min(max(args.steps, 20), 200)

    def time_calls(fn, clock_name: str | None = None, reps: int = reps, settle: float = 0.0) -> float:
        """Average device time of one call: `reps` calls captured in a CUDA graph and replayed once, so
        host-side launch cost does not enter (plain back-to-back calls when capture fails).  With
        settle, an idle pause comes first; with clock_name, the clocks are sampled over exactly that
        replay (rank 0) and the summary is kept in kernel_clocks[clock_name]."""
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g = None
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(reps):
                    fn()
            g.replay()
            torch.cuda.synchronize()
        except Exception:
            g = None
            torch.cuda.synchronize()

        def run_once():
            if g is not None:
                g.replay()
            else:
                for _ in range(reps):
                    fn()

        if settle > 0:
            time.sleep(settle)  # an idle pause, so a short (burst) measurement starts from rested clocks
        smp = ClockSampler(uuid) if (clock_name and rank == 0) else None
        if smp is not None:
            smp.start()
            time.sleep(0.05)  # the sampler's first readings
        th0 = time.time()
        a.record(stream)
        run_once()
        b.record(stream)
        torch.cuda.synchronize()
        total_ms = a.elapsed_time(b)
        if smp is not None:
            smp.mark(th0, time.time())
            kernel_clocks[clock_name] = smp.stop()
        del g
        return total_ms / reps

    kernel_clocks = {}
    # the dominant kernel pair, timed alone with its own clock record: as many back-to-back calls as
    # the timed region has steps (against the burst peak while the loop ends before the power cap's
    # onset, else the sustained one), and a 200-call loop of about 0.3 s (the power-capped regime)
    ffn_reps = max(20, args.steps)
    ms_ffn = time_calls(lambda: buf.expert_ffn(True), clock_name="ffn", reps=ffn_reps, settle=0.5)
    # the small stages, each after an idle pause: a latency-bound kernel timed right after a power-capped
    # GEMM loop would be measured at the capped clock
    ms_route = time_calls(buf.route, settle=0.3)
    ms_permute = time_calls(buf.permute, settle=0.3)
    # standalone combine (the unfused path: y materialised by moe_expert_ffn(fuse_combine=0))
    buf.permute()
    buf.expert_ffn(False)
    ms_combine = time_calls(buf.combine, settle=0.3)
    ms_ffn_sus = time_calls(lambda: buf.expert_ffn(True), clock_name="ffn_sustained", reps=200, settle=0.3)
    buf.forward()
    torch.cuda.synchronize()
    counts = buf.expert_counts.cpu().numpy()
    kept = int(counts.sum())
    touched = int((counts > 0).sum())
    drops = int(buf.dropped.cpu().numpy().sum())
    losses = buf.losses.cpu().numpy()

    # losses of the whole job's batch: every replica's loss sums all-reduced (one small collective,
    # outside the timed regions; with one GPU these are this batch's own losses)
    buf.forward()
    global_losses = buf.global_losses().cpu().numpy()

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    ffn_flops = 4.0 * cfg.H * cfg.F * kept
    tflops = ffn_flops / (ms_ffn / 1000.0) / 1e12
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    router_bytes = cfg.T * cfg.H * es + cfg.H * cfg.E * es + cfg.T * cfg.k * 8
    # permute: read the kept x rows, write them to x_perm, clear out (fp32), index traffic
    permute_bytes = kept * cfg.H * es * 2 + cfg.T * cfg.H * 4 + cfg.T * cfg.k * 8
    # combine: read every kept row of y (fp32), write out (fp32), index and weight traffic
    combine_bytes = kept * cfg.H * 4 + cfg.T * cfg.H * 4 + cfg.T * cfg.k * 8
    traffic = None
    # ---------------- training step: forward that keeps state + backward (bf16 token choice) -----
    train = None
    if not args.no_train and cfg.dtype == "bf16" and cfg.routing == "token_choice":
        tbuf = moe.MoEBuffers(shape, dev, train=True)
        grads = tbuf.make_grads(with_dw=False)
        dout = torch.randn((cfg.T, cfg.H), dtype=torch.float32, device="cuda",
                           generator=torch.Generator(device="cuda").manual_seed(cfg.seed))
        tbuf.forward_train()
        ms_fwd_train = time_calls(tbuf.forward_train)
        ms_bwd = time_calls(lambda: tbuf.backward(dout, grads, 0.01, 0.001), clock_name="bwd", reps=100)
        bwd_launches = moe.moe_last_launch_count()
        tkept = int(tbuf.expert_counts.sum().item())
        bwd_flops = 8.0 * cfg.H * cfg.F * tkept + 4.0 * cfg.T * cfg.H * cfg.E
        train = {"fwd_train_ms": ms_fwd_train, "bwd_ms": ms_bwd, "step_ms": ms_fwd_train + ms_bwd,
                 "tokens_per_s": cfg.T / ((ms_fwd_train + ms_bwd) / 1000.0),  # rank 0's replica
                 "bwd_tflops": bwd_flops / (ms_bwd / 1000.0) / 1e12,
                 "bwd_frac_burst": bwd_flops / (ms_bwd / 1000.0) / 1e12 / peaks["bf16_tflops"],
                 "bwd_frac_sustained": bwd_flops / (ms_bwd / 1000.0) / 1e12 / peaks["bf16_tflops_sustained"],
                 "bwd_clocks": kernel_clocks.get("bwd"),
                 "bwd_launches": bwd_launches,
                 "note": "backward = dout row gather, dgrad W2 (+du, dw), dgrad W1 (+dx), wgrad W2, wgrad W1, bias "
                         "gradients, router backward, gate weight gradient; flops 8*H*F per kept row + 4*T*H*E"}
        del tbuf, grads, dout
        torch.cuda.empty_cache()

    traffic = captured_traffic(cfg.name)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_rate(cfg, inp, budget_s=args.cpu_budget)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": workload_config(cfg), "global_batch": world * cfg.T, "seq_len": None,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: the expert weights (%.2f GB) stream every step" %
                         (cfg.E * 2 * cfg.H * cfg.F * es / 1e9)},
        "roofline": dict(ffn_roofline(cfg, kept, touched, ms_ffn, peaks, None, sms, ffn_reps * ms_ffn / 1000.0),
                         traffic=traffic, clocks=kernel_clocks.get("ffn"), calls_timed=ffn_reps,
                         clocks_note="NVML refreshes the SM clock reading about every 100 ms and power later "
                                     "still, so over a loop of a few tens of milliseconds the record shows the "
                                     "state before the power cap responds; the per-SM-cycle rate is given for "
                                     "the sustained loop, whose clock record is steady",
                         sustained=sustained_roofline(cfg, kept, ms_ffn_sus, peaks, kernel_clocks.get("ffn_sustained"),
                                                      sms),
                         kernel="grouped GEMMs (GEMM1 bias+act, GEMM2 scale+combine), one moe_expert_ffn call"),
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": cfg.T * cfg.H * es,
                "d2h_bytes_per_step": cfg.T * cfg.H * 4, "api": "moe_forward_host",
                "mode": f"pipelined: {NBUF} buffer sets on {NBUF} streams, steps rotate", "serial_value": e2e_serial,
                "max_abs_diff_across_buffer_sets": out_diff, "device_status": e2e_status},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "kernels": {
            "ffn_ms": ms_ffn, "route_ms": ms_route, "permute_ms": ms_permute,
            "ffn_tflops": tflops, "ffn_frac_burst_peak": tflops / peaks["bf16_tflops"],
            "ffn_frac_nominal_2250": tflops / 2250.0,
            "route_gbs": router_bytes / (ms_route / 1000.0) / 1e9,
            "permute_gbs": permute_bytes / (ms_permute / 1000.0) / 1e9,
            "combine_ms": ms_combine,
            "combine_gbs": combine_bytes / (ms_combine / 1000.0) / 1e9,
            "hbm_peak_gbs": peaks["hbm_gbs"],
            "layer_roofline_ms": 1000 * max(alg_flops(cfg, kept) / (peaks["bf16_tflops"] * 1e12),
                                            alg_bytes(cfg, touched) / (peaks["hbm_gbs"] * 1e9)),
        },
        "train": train,
        "layer": {"kept": kept, "dropped": drops, "touched_experts": touched, "aux_loss": float(losses[0]),
                  "z_loss": float(losses[1]), "expert_counts_min_max": [int(counts.min()), int(counts.max())],
                  "global_aux_loss": float(global_losses[0]), "global_z_loss": float(global_losses[1])},
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="mixtral", choices=list(synth.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-train", action="store_true", help="skip the training-step (forward + backward) timing")
    ap.add_argument("--cpu-budget", type=float, default=30.0, help="seconds of oracle time for cpu_baseline")
    for dim in ("T", "H", "E", "k", "F"):
        ap.add_argument(f"--{dim}", type=int, default=None, help=f"override {dim} of the workload (profiling)")
    args = ap.parse_args()
    cfg = synth.CONFIGS[args.config]
    over = {d: getattr(args, d) for d in ("T", "H", "E", "k", "F") if getattr(args, d) is not None}
    if over:
        cfg = cfg.with_(name=cfg.name + "[" + ",".join(f"{d}={v}" for d, v in over.items()) + "]", **over)
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours_impl(args, cfg)


if __name__ == "__main__":
    main()
