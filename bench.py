#!/usr/bin/env python
"""Bench: KDA forward (prefill) throughput on B200, in Mtok*head/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl kda|reference]

A step is one kda_fwd call over the whole workload (every (sequence, head)
chain of the batch), i.e. the full hot path. The default workload is the
Kimi-Linear-shaped fixed-length batch (T = 8192, H = 32, d = 128, zero initial
state, final state returned). Inputs are seeded synthetic data of that shape
(kda_inputs). For N > 1 (torchrun) every rank runs its own independent batch
(weak scaling, no data-path collective); the time is the max over ranks.

Output: one JSON line on rank 0 (see the keys in ``main``).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import kda_inputs  # noqa: E402

METRIC = "KDA fwd prefill Mtok·head/s at d=128 on 1 B200; % of TC/HBM roofline"
UNIT = "Mtok·head/s"
D = 128
# Counted work per token*head (d = 128): q, k, v, o bf16 + g fp32 + beta fp32.
BYTES_PER_TOKHEAD = 3 * D * 2 + D * 4 + 4 + D * 2          # 1540 B
FLOPS_PER_TOKHEAD = 6 * D * D + 10 * 16 * D                # 118784 FLOP
STATE_BYTES = D * D * 4                                    # one (sequence, head) state
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CSRC = os.path.join(ROOT, "kimi_delta_attention_26_b200", "csrc")
KERNEL_SOURCES = [os.path.join(CSRC, f)
                  for f in ("kda_prims.cuh", "kda_fwd16.cuh", "kda_fwd64.cuh", "kda_split.cuh", "kda_decode.cuh",
                            "kda_bwd.cuh", "kda_api.cu")]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def _code_only(src: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace collapsed, so
    that editing a comment does not count as changing the kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif src[i] in "\"'":
            q, j = src[i], i + 1
            while j < n and src[j] != q:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return " ".join("".join(out).split())


def kernel_source_sha(names=None) -> str:
    """Hash of the kernels' code (comments and layout excluded) over the named
    csrc files (default: all): a profile's DRAM traffic applies while this
    matches the hash recorded with it."""
    paths = KERNEL_SOURCES if not names else [os.path.join(CSRC, n) for n in names]
    h = hashlib.sha256()
    for p in paths:
        with open(p, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def recorded_traffic(profile: str):
    """DRAM bytes per launch from the committed ncu summary
    profiles/<profile>.md, if it was taken on the current source of the
    kernels it names (else None)."""
    p = os.path.join(ROOT, "profiles", f"{profile}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_b = re.search(r"traffic_bytes_per_launch\s*=\s*([0-9.eE+]+)", txt)
    m_s = re.search(r"kernel_source_sha256\s*=\s*([0-9a-f]{64})", txt)
    m_n = re.search(r"kernel_sources\s*=\s*([\w. ]+)", txt)
    names = m_n.group(1).split() if m_n else None
    if not m_b or not m_s or m_s.group(1) != kernel_source_sha(names):
        return None
    return float(m_b.group(1))


def work_units(inp) -> int:
    return inp.total_tokens * inp.num_heads


def algorithmic_bytes(inp, with_init: bool, with_final: bool) -> int:
    n = work_units(inp) * BYTES_PER_TOKHEAD
    states = inp.num_seqs * inp.num_heads * STATE_BYTES
    return n + (states if with_init else 0) + (states if with_final else 0)


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = 0
        self.ok = False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            bus = None
            try:
                import torch

                props = torch.cuda.get_device_properties(device_index)
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            log(f"clock sampling unavailable: {e}")
        self.period = period_s
        self._t = None

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        self.reasons |= int(r)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------ CPU (oracle) leg
def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_prefix_run(inp, ntok: int, nthreads: int) -> float:
    """Run the oracle (as it stands) on the first ntok tokens of every sequence
    prefix of the packed batch; returns seconds."""
    import oracle  # test infrastructure; only this leg of the bench executes it

    ntok = max(1, min(ntok, inp.total_tokens))
    cu = np.minimum(inp.cu_seqlens, ntok).astype(np.int32)
    init = inp.initial_state
    t = time.perf_counter()
    oracle.scan(inp.q[:ntok], inp.k[:ntok], inp.v[:ntok], inp.g[:ntok], inp.beta[:ntok], cu, inp.scale, init,
                nthreads=nthreads)
    return time.perf_counter() - t


def cpu_baseline(inp, target_s: float):
    """Time the oracle on a bounded sample: a token prefix sized for about
    target_s seconds, repeated (whole workload) when the workload is smaller."""
    nthreads = cpu_threads()
    probe = min(inp.total_tokens, 64)
    t_probe = oracle_prefix_run(inp, probe, nthreads)
    ntok = int(min(inp.total_tokens, max(probe, probe * target_s / max(t_probe, 1e-6))))
    dt, reps = 0.0, 0
    while reps == 0 or (dt < target_s and reps < 50):
        dt += oracle_prefix_run(inp, ntok, nthreads)
        reps += 1
    units = ntok * inp.num_heads * reps
    return {"value": units / dt / 1e6, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"fp64 token scan on the first {ntok} of {inp.total_tokens} tokens, all "
                      f"{inp.num_heads} heads, {reps} pass(es) ({units} tok*head, {dt:.1f} s, {nthreads} threads)"}


# ----------------------------------------------------------------- dist utils
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(times_ms, units):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    t = max(times_ms)
    return sum(units) / (t * 1e-3) / 1e6, t


def reduce_over_ranks(ms: float, e2e_ms: float, units: float, device=None):
    """Max of the per-rank times and sum of the per-rank work units over the
    default process group (NCCL on GPUs, gloo on CPU). Returns
    (ms, e2e_ms, total_units); identity without a process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms, e2e_ms, float(units)
    tt = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    uu = torch.tensor([float(units)], dtype=torch.float64, device=device)
    dist.all_reduce(uu)
    return float(tt[0]), float(tt[1]), float(uu[0])


# ---------------------------------------------------------------- reference
def input_bytes(inp) -> int:
    """Bytes of the inputs the kernel reads (q, k, v, g, beta, cu_seqlens and
    the initial state when there is one)."""
    arrs = [inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens]
    if inp.initial_state is not None:
        arrs.append(inp.initial_state)
    return int(sum(a.nbytes for a in arrs))


def workload_config(wl, inp, ws: int) -> dict:
    """The `config` object of both arms' JSON lines for this workload."""
    in_bytes = input_bytes(inp)
    T, H, N = inp.total_tokens, inp.num_heads, inp.num_seqs
    return {"workload": wl.name, "seq_lens": list(wl.seqlens) if len(wl.seqlens) <= 16 else None,
            "total_tokens": T, "num_heads": H, "head_dim": D, "num_seqs": N,
            "initial_state": "random" if inp.initial_state is not None else "zero", "final_state": True,
            "global_batch": N * ws, "seq_len": T,
            "l2": "flushed between launches" if in_bytes < 2 * L2_BYTES
                  else f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB)",
            "parallelism": f"dp{ws} (independent batch per GPU)", "seed": wl.seed}


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0  # the CPU oracle arm runs on rank 0 only
    wl = kda_inputs.workload(args.config)
    inp = wl.make()
    nthreads = cpu_threads()
    budget = min(10.0, 150.0 / max(1, args.steps + args.warmup))
    probe = min(inp.total_tokens, 64)
    t_probe = oracle_prefix_run(inp, probe, nthreads)
    ntok = int(min(inp.total_tokens, max(probe, probe * budget / max(t_probe, 1e-6))))
    for _ in range(args.warmup):
        oracle_prefix_run(inp, ntok, nthreads)
    dts = [oracle_prefix_run(inp, ntok, nthreads) for _ in range(args.steps)]
    dt = sum(dts) / len(dts)
    units = ntok * inp.num_heads
    value = units / dt / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, inp, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": f"fp64 token scan on the first {ntok} of {inp.total_tokens} tokens, "
                                   f"all {inp.num_heads} heads, per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0



def hide_host_latency(stream, cycles: int = 400_000):
    """Keep the device busy (~0.2 ms) while the host prepares the next launch,
    so that the start event and the kernel run back to back on the device:
    the timed interval then holds device time only, not the binding's host
    work between the two enqueues."""
    import torch

    with torch.cuda.stream(stream):
        torch.cuda._sleep(cycles)


def roofline_fields(inp, ms: float, with_init: bool, wl_name: str):
    """Throughput and roofline figures of one launch of `ms` milliseconds."""
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    units = work_units(inp)
    bytes_launch = algorithmic_bytes(inp, with_init, True)
    flops_launch = units * FLOPS_PER_TOKHEAD
    gbs = bytes_launch / (ms * 1e-3) / 1e9
    tflops = flops_launch / (ms * 1e-3) / 1e12
    t_hbm = bytes_launch / (hbm_peak * 1e9)
    t_tc = flops_launch / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    roof = {"bound": bound,
            "achieved": gbs if bound == "hbm" else tflops,
            "peak": hbm_peak if bound == "hbm" else tc_peak,
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "peak_source": f"{peak_kind} ({'MEASURED_PEAKS.json' if peak_kind == 'measured' else 'recipe fallback'})",
            "traffic": recorded_traffic(f"kda_fwd_{wl_name}"),
            "algorithmic_bytes_per_launch": bytes_launch,
            "tflops_counted": tflops}
    roof["frac"] = roof["achieved"] / roof["peak"]
    return roof


def time_launches(launch, steps: int, warmup: int, stream, flush, dev):
    """Per-launch device times (ms) of `steps` launches on `stream`, after
    `warmup` untimed ones, with an L2 flush before each timed launch."""
    import torch

    for _ in range(warmup):
        launch()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.add_(1.0)
        hide_host_latency(stream)
        ev[i][0].record(stream)
        launch()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    return [a.elapsed_time(b) for a, b in ev]


def per_config_table(kda, dev, stream, steps: int, paths):
    """Every workload, each kernel path: device time per launch (inputs
    resident, L2 flushed between launches) and the roofline figures."""
    import torch

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    table = {}
    for cfg in sorted(kda_inputs.WORKLOADS):
        wl = kda_inputs.workload(cfg)
        inp = wl.make()
        t = lambda a: torch.from_numpy(a).to(dev)
        q, k, v = (t(x).view(torch.bfloat16) for x in (inp.q, inp.k, inp.v))
        g, beta, cu = t(inp.g), t(inp.beta), t(inp.cu_seqlens)
        init = None if inp.initial_state is None else t(inp.initial_state)
        out = torch.empty_like(q)
        fin = torch.empty((inp.num_seqs, inp.num_heads, D, D), dtype=torch.float32, device=dev)
        row = {"workload": wl.name, "config": cfg, "tokens": inp.total_tokens, "heads": inp.num_heads}
        for path in paths:
            kda.set_path(path)
            launch = lambda: kda.kda_fwd(q, k, v, g, beta, inp.scale, cu, init, out=out, final_state=fin,
                                         stream=stream)
            ms_l = time_launches(launch, steps, 3, stream, flush, dev)
            ms = sum(ms_l) / len(ms_l)
            roof = roofline_fields(inp, ms, init is not None, wl.name if path == 0 else f"{wl.name}_p{path}")
            row[f"path{path}" if path else "default"] = {
                "ms": ms, "value": work_units(inp) / (ms * 1e-3) / 1e6, "unit": UNIT,
                "roofline_frac": roof["frac"], "gbs": roof["achieved"] if roof["bound"] == "hbm" else None,
                "tflops_counted": roof["tflops_counted"], "traffic": roof["traffic"],
                "algorithmic_bytes_per_launch": roof["algorithmic_bytes_per_launch"]}
        kda.set_path(0)
        table[wl.name] = row
        del q, k, v, g, beta, cu, init, out, fin
    return table


def decode_entry(kda, dev, stream, steps: int):
    """The decode step (one token for each of 256 requests, H=32, states
    resident and updated in place): device time per launch and its HBM
    roofline (the step reads and writes every state once)."""
    import torch

    wl = kda_inputs.DECODE
    inp = wl.make()
    t = lambda a: torch.from_numpy(a).to(dev)
    q, k, v = (t(x).view(torch.bfloat16) for x in (inp.q, inp.k, inp.v))
    g, beta, state = t(inp.g), t(inp.beta), t(inp.initial_state)
    out = torch.empty_like(q)
    launch = lambda: kda.kda_decode(q, k, v, g, beta, state, scale=inp.scale, out=out, stream=stream)
    # the states (512 MiB) exceed L2, so launches need no flush between them
    ms_l = time_launches(launch, steps, 3, stream, None, dev)
    ms = sum(ms_l) / len(ms_l)
    hbm_peak, _, peak_kind = measured_peaks()
    units = work_units(inp)
    bytes_launch = units * (BYTES_PER_TOKHEAD + 2 * STATE_BYTES)
    gbs = bytes_launch / (ms * 1e-3) / 1e9
    return {"workload": wl.name, "requests": inp.num_seqs, "heads": inp.num_heads, "ms": ms,
            "value": units / (ms * 1e-3) / 1e6, "unit": UNIT,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "peak_source": peak_kind, "algorithmic_bytes_per_launch": bytes_launch,
                         "traffic": recorded_traffic(f"kda_decode_{wl.name}")},
            "l2": "states (512 MiB) larger than L2"}


def fused_entry(kda, dev, stream, steps: int):
    """kda_fwd_fused on the Kimi-Linear-shaped workload (T=8192, H=32) from
    the raw draws (q, k unnormalised, gate and beta logits): device time per
    launch, L2 flushed between launches, and its HBM roofline (the same
    bytes per token and head as kda_fwd)."""
    import torch

    wl = kda_inputs.workload(2)
    inp = wl.make(raw=True)
    t = lambda a: torch.from_numpy(a).to(dev)
    q, k, v = (t(x).view(torch.bfloat16) for x in (inp.q_raw, inp.k_raw, inp.v))
    g, beta = t(inp.g_logit), t(inp.beta_logit)
    out = torch.empty_like(q)
    fin = torch.empty((inp.num_seqs, inp.num_heads, D, D), dtype=torch.float32, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    launch = lambda: kda.kda_fwd_fused(q, k, v, g, beta, inp.scale, -5.0, out=out, final_state=fin, stream=stream)
    ms_l = time_launches(launch, steps, 3, stream, flush, dev)
    ms = sum(ms_l) / len(ms_l)
    roof = roofline_fields(inp, ms, False, f"{wl.name}_fused")
    return {"workload": wl.name + " (raw q/k, gate and beta logits)", "ms": ms,
            "value": work_units(inp) / (ms * 1e-3) / 1e6, "unit": UNIT, "roofline_frac": roof["frac"],
            "gbs": roof["achieved"], "traffic": roof["traffic"],
            "algorithmic_bytes_per_launch": roof["algorithmic_bytes_per_launch"]}


# The backward's algorithmic work per token and head: one forward step
# (decay, S'^T k, write: 5 flops per state element) and one reverse step
# (20 flops per state element: the rank-1 updates and reductions of the
# reverse recurrence) over the 128 x 128 state. Its bytes: the inputs, dO,
# and the fp32 gradients of q, k, v, g and beta.
BWD_FLOPS_PER_TOKHEAD = 25 * D * D
BWD_BYTES_PER_TOKHEAD = 3 * D * 2 + D * 4 + 4 + D * 2 + 4 * D * 4 + 4
# fp32 FMA issue of the CUDA cores: 148 SMs x 128 lanes x 2 flops per cycle at
# the 1965 MHz maximum SM clock (the backward's rank-1 updates run there)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_entry(kda, dev, stream, steps: int, tokens: int = 8192):
    """kda_bwd on the Kimi-Linear-shaped workload (T=8192, H=32; `tokens`
    shortens it, for profiling captures) with a random output gradient: device
    time per launch (L2 flushed between launches) and its roofline on the fp32
    CUDA cores."""
    import torch

    wl = kda_inputs.workload(2)
    inp = kda_inputs.make_inputs([tokens], wl.num_heads, wl.seed) if tokens != wl.total_tokens else wl.make()
    t = lambda a: torch.from_numpy(a).to(dev)
    q, k, v = (t(x).view(torch.bfloat16) for x in (inp.q, inp.k, inp.v))
    g, beta = t(inp.g), t(inp.beta)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    dout = torch.randn(q.shape, device=dev, generator=gen).bfloat16()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    launch = lambda: kda.kda_bwd(q, k, v, g, beta, dout, inp.scale, stream=stream)
    ms_l = time_launches(launch, steps, 3, stream, flush, dev)
    ms = sum(ms_l) / len(ms_l)
    units = work_units(inp)
    tflops = units * BWD_FLOPS_PER_TOKHEAD / (ms * 1e-3) / 1e12
    gbs = units * BWD_BYTES_PER_TOKHEAD / (ms * 1e-3) / 1e9
    name = wl.name if tokens == wl.total_tokens else f"fixed_T{tokens}_H{wl.num_heads}"
    return {"workload": name + " (gradients of q, k, v, g, beta)", "ms": ms,
            "value": units / (ms * 1e-3) / 1e6, "unit": UNIT,
            "roofline": {"bound": "alu", "achieved": tflops, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                         "frac": tflops / FP32_ALU_TFLOPS,
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz",
                         "algorithmic_flops_per_launch": units * BWD_FLOPS_PER_TOKHEAD},
            "gbs": gbs}


# ---------------------------------------------------------------------- kda
def run_kda(args):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    if ws != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE={ws}; using WORLD_SIZE")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    import kimi_delta_attention_26_b200 as kda

    kda.set_path(args.path)
    if args.only:
        st = torch.cuda.current_stream(dev)
        if rank == 0:
            if args.only == "backward":
                res = bwd_entry(kda, dev, st, args.steps, args.bwd_tokens)
            else:
                res = {"decode": decode_entry, "fused": fused_entry}[args.only](kda, dev, st, args.steps)
            print(json.dumps(res), flush=True)
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    wl = kda_inputs.workload(args.config)
    inp = wl.make(seed=wl.seed + rank)  # an independent batch per rank
    with_init = inp.initial_state is not None
    stream = torch.cuda.current_stream(dev)

    # pinned host copies (for the end-to-end leg) and device-resident inputs
    def pinned(a):
        return torch.from_numpy(a).pin_memory()

    h = {"q": pinned(inp.q).view(torch.bfloat16), "k": pinned(inp.k).view(torch.bfloat16),
         "v": pinned(inp.v).view(torch.bfloat16), "g": pinned(inp.g), "beta": pinned(inp.beta),
         "cu": pinned(inp.cu_seqlens)}
    if with_init:
        h["init"] = pinned(inp.initial_state)
    d = {key: t.to(dev, non_blocking=False) for key, t in h.items()}
    T, H, N = inp.total_tokens, inp.num_heads, inp.num_seqs
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    fin = torch.empty((N, H, D, D), dtype=torch.float32, device=dev)
    h_out = torch.empty((T, H, D), dtype=torch.bfloat16).pin_memory()
    h_fin = torch.empty((N, H, D, D), dtype=torch.float32).pin_memory()

    in_bytes = sum(t.numel() * t.element_size() for t in d.values())
    assert in_bytes == input_bytes(inp)
    flush = None
    if in_bytes < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu"], d.get("init"),
                    out=out, final_state=fin, stream=stream)

    def barrier():
        if ws > 1:
            dist.barrier()

    # ---- device-resident timing: per-launch CUDA events on the launch stream
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        if flush is not None:
            flush.add_(1.0)  # evict the previous launch's working set from L2
        hide_host_latency(stream)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.stop()
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    ms = sum(launch_ms) / len(launch_ms)

    # ---- end-to-end through the public API with host buffers
    def e2e_step():
        for key in d:
            d[key].copy_(h[key], non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)
        h_fin.copy_(fin, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 3))):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 10))
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    h2d = in_bytes
    d2h = h_out.numel() * h_out.element_size() + h_fin.numel() * h_fin.element_size()

    # ---- max over ranks
    units = work_units(inp)
    ms, e2e_ms, total_units = reduce_over_ranks(ms, e2e_ms, units, device=dev)
    value = total_units / (ms * 1e-3) / 1e6
    e2e_value = total_units / (e2e_ms * 1e-3) / 1e6

    if rank == 0:
        roof = roofline_fields(inp, ms, with_init, wl.name)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(wl, inp, ws),
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": args.steps,
            "launch_ms": {"min": min(launch_ms), "median": statistics.median(launch_ms), "max": max(launch_ms)},
            "clocks": sampler.summary(),
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(inp, args.cpu_seconds)
        if ws == 1 and not args.no_per_config:
            # the extra entries never cost the headline line: a failure is recorded in its place
            extras = [("per_config", lambda: per_config_table(kda, dev, stream, min(args.steps, 20), (0, 64))),
                      ("decode", lambda: decode_entry(kda, dev, stream, min(args.steps, 20))),
                      ("fused_gate", lambda: fused_entry(kda, dev, stream, min(args.steps, 20))),
                      ("backward", lambda: bwd_entry(kda, dev, stream, min(args.steps, 5)))]
            for key, fn in extras:
                try:
                    line[key] = fn()
                except Exception as e:  # reported, not hidden: the value names the failure
                    log(f"{key} entry failed: {e!r}")
                    line[key] = {"error": repr(e)}
                    kda.set_path(args.path)
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2, choices=sorted(kda_inputs.WORKLOADS))
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload table (every workload, both kernel paths)")
    ap.add_argument("--only", choices=["decode", "fused", "backward"],
                    help="time only that entry (decode step, fused-preprocessing prefill or backward) and print its "
                         "JSON object")
    ap.add_argument("--bwd-tokens", type=int, default=8192,
                    help="sequence length of the backward entry (H=32); shorter for profiling captures")
    ap.add_argument("--path", type=int, default=0, choices=[0, 16, 64],
                    help="kernel: 0 = library default (16-token chunks on mma.sync, time split where it wins), "
                         "16 = 16-token chunks, 64 = 64-token chunks on tcgen05")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        log("note: raising --warmup to 3 (minimum)")
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_kda(args)


if __name__ == "__main__":
    sys.exit(main())
