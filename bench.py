"""LatentMoE layer forward benchmark: tokens/s on B200 and the dominant kernel's roofline fraction.

One step = one full layer forward (router GEMM, top-K' + softmax, counting
sort, expert up / down GEMMs, combine, up-projection + residual) over one
batch of seeded synthetic tokens, with weights and inputs resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference] [--ep]

Prints one JSON line (rank 0).  Under torchrun (N > 1) every rank runs an
independent replica of the layer on its own tokens (the layer shards by
tokens with no exchange step), so per-GPU work is fixed: weak scaling.
With --ep the ranks instead split the FFN experts (expert parallelism): each
rank routes its own tokens and the latent rows cross ranks by NCCL all-to-all
before and after the experts; with one rank nothing moves and the step times
the three stages of that forward alone.

The timed steps are plain lmoe_forward calls (each forward reaches the GPU as
the library's own CUDA graph); `graph_replay` adds the same steps replayed from
graphs captured by the caller.  SM clocks and throttle reasons are sampled
through NVML while the timed steps run.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from latent_mixture_experts_gemm_b200 import lmoe, synth  # noqa: E402

METRIC = "LatentMoE layer tokens/s at 1 B200 (prefill & decode); % of BF16/HBM roofline"
DEFAULT_WORKLOAD = "nemotron_decode"
#: the other layer configurations, each measured in the same run and reported under `secondary`: the
#: Nemotron-like prefill, the standard MoE at equal budget (prefill and decode), the Kimi-like skewed layer
#: with MoE++ experts, and the Nemotron-like decode batch with NVFP4 and MXFP4 expert weights
SECONDARY_WORKLOADS = ("nemotron_prefill", "std_prefill", "std_decode", "kimi_skew", "nemotron_decode_nvfp4",
                       "nemotron_decode_mxfp4")
N_INPUT_BATCHES = 4  # distinct token batches cycled through the steps


# ----------------------------------------------------------------------------- peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
# Throttle reasons reported in the clock record, with the NVML constant of each.
CLOCK_REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
                 ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
                 ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
                 ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))


def clock_summary(samples, max_mhz, nvml):
    """The clock record from (SM MHz, reason bits) samples: the median clock, the maximum clock and the names
    of the reasons any sample had active."""
    reasons = sorted(name for name, const in CLOCK_REASONS
                     if any(bits & getattr(nvml, const) for _, bits in samples))
    sm = [mhz for mhz, _ in samples]
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max_mhz, "reasons": reasons,
            "samples": len(sm)}


class ClockSampler:
    """SM clock and throttle reasons sampled while the timed region runs (read-only queries).

    NVML, the library nvidia-smi reads, is polled every 0.5 ms from a thread, so even the ~6 ms of 20 decode
    steps get a dozen samples.  While it runs, the interpreter hands the GIL over every 0.1 ms instead of its
    default 5 ms, so the polling thread is not starved by the launching one.  Without NVML, nvidia-smi runs
    every 200 ms instead.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.0005

    def __init__(self, device_uuid: str):
        self.uuid = device_uuid
        self.proc = None
        self.lines = []
        self.thread = None
        self.nvml = None
        self.handle = None
        self.samples = []
        self.done = threading.Event()
        self.switch = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            # the first queries after initialisation are slow (milliseconds): make them before the timed region
            pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            self.nvml = pynvml
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _poll(self):
        n = self.nvml
        while not self.done.is_set():
            try:
                mhz = float(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
                bits = int(n.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
                self.samples.append((mhz, bits))
            except Exception:
                return
            time.sleep(self.PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.done.set()
            if self.thread:
                self.thread.join(timeout=2)
            if self.switch is not None:
                sys.setswitchinterval(self.switch)
            try:
                max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
            except Exception:
                max_mhz = None
            out = clock_summary(self.samples, max_mhz, self.nvml)
            out["source"] = "nvml, every 0.5 ms"
            return out
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, every 200 ms"}


def _smi_id(device: int) -> str:
    """nvidia-smi --id for a torch device (its UUID; CUDA_VISIBLE_DEVICES may renumber indices)."""
    try:
        u = str(torch.cuda.get_device_properties(device).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(device)


# ----------------------------------------------------------------------------- ranks
def dist_barrier(world: int) -> None:
    """Barrier over all ranks (no-op for one process)."""
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()


def dist_max(v: float, world: int, device: torch.device) -> float:
    """Maximum of a per-rank value over all ranks (the job's time is the slowest rank's)."""
    if world <= 1:
        return v
    import torch.distributed as tdist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- algorithmic work
#: bytes per stored expert weight: bf16; MXFP8 (E4M3 + one E8M0 byte per 32); MXFP4 (E2M1 + one per 32);
#: NVFP4 (E2M1 + one E4M3 byte per 16; the fp32 scale per expert matrix is negligible)
WEIGHT_BYTES = {0: 2.0, 1: 1.0 + 1.0 / 32, 2: 0.5 + 1.0 / 32, 3: 0.5 + 1.0 / 16}
#: bytes per element of the expert GEMMs' token operands (MXFP8 with MX experts, NVFP4 with NVFP4 experts)
ACT_BYTES = {0: 2.0, 1: 1.0 + 1.0 / 32, 2: 1.0 + 1.0 / 32, 3: 0.5 + 1.0 / 16}
#: tensor-core rate of the expert GEMMs relative to bf16: the nominal fp8 : bf16 ratio (4.5 : 2.25) for the
#: MX kinds (E2M1 weights meet E4M3 inputs there), fp4 : bf16 (9 : 2.25) for NVFP4
EXPERT_RATE = {0: 1.0, 1: 2.0, 2: 2.0, 3: 4.0}


#: DRAM bytes (read + write) per launch of each workload's expert phases, from ncu captures of the kernels as
#: they are now (dram__bytes_read.sum + dram__bytes_write.sum): decode streams as the mean over the captured
#: steps' launches, prefill grouped GEMMs from one launch each at the full token count.  A kernel that changes
#: drops out of this table until it is captured again.
NCU_TRAFFIC = {
    ("nemotron_decode", "expert_up_stream"): 797.8e6,
    ("nemotron_decode", "expert_down_stream"): 797.8e6,
    ("nemotron_prefill", "expert_up_gemm"): 1792.1e6,
    ("nemotron_prefill", "expert_down_gemm"): 1788.5e6,
    ("std_decode", "expert_up_stream"): 836.5e6,
    ("std_decode", "expert_down_stream"): 839.2e6,
    ("std_prefill", "expert_up_gemm"): 1662.7e6,
    ("std_prefill", "expert_down_gemm"): 1554.5e6,
    ("kimi_skew", "expert_up_gemm"): 1237.9e6,
    ("kimi_skew", "expert_down_gemm"): 772.3e6,
    ("nemotron_decode_nvfp4", "expert_up_stream"): 229.7e6,
    ("nemotron_decode_nvfp4", "expert_down_stream"): 230.0e6,
    ("nemotron_decode_mxfp4", "expert_up_stream"): 214.2e6,
    ("nemotron_decode_mxfp4", "expert_down_stream"): 214.4e6,
}


def layer_work(cfg, stats, T):
    """F (FLOPs), B (bytes) and F_eff (FLOPs at the bf16 rate that take as long) of one forward, from its actual
    routing (plus the shared expert, if any)."""
    g = 2 if cfg.gated else 1
    fmt = getattr(cfg, "expert_fmt", 0)
    wb = WEIGHT_BYTES[fmt]
    R, E = stats["ffn_rows"], stats["experts_touched"]
    d, L, m, nt = cfg.d, cfg.latent, cfg.m, cfg.n_total
    fe = 2 * (g + 1) * (L if cfg.has_proj else d) * m * R  # expert FLOPs
    if cfg.has_proj:
        F = 2 * T * (2 * d * L + d * nt)
        B = wb * (g + 1) * L * m * E + 2 * (2 * d * L + d * nt) + 2 * 2 * T * d
    else:
        F = 2 * T * d * nt
        B = wb * (g + 1) * d * m * E + 2 * d * nt + 4 * T * d
    ms = getattr(cfg, "shared_m", 0)
    if ms:
        F += 2 * T * (g + 1) * d * ms
        B += 2 * (g + 1) * d * ms
    F_eff = F + fe / EXPERT_RATE[fmt]
    return float(F + fe), float(B), float(F_eff)


def phase_units(cfg, stats, T, phase):
    """Algorithmic (flops, bytes) of one launch of a phase's kernel.

    The expert phases count the weights of the experts they touch as their bytes: the gathered rows they read
    and the hidden rows / expert outputs they write are the layer's intermediates, implementation traffic like
    the ncu `traffic` figure, not algorithmic bytes.  So a grouped GEMM on a prefill batch is tensor-bound
    (thousands of FLOPs per weight byte), and a weight stream on a decode batch HBM-bound."""
    g = 2 if cfg.gated else 1
    d, L, m, nt = cfg.d, cfg.latent, cfg.m, cfg.n_total
    fmt = getattr(cfg, "expert_fmt", 0)
    wb, ab = WEIGHT_BYTES[fmt], ACT_BYTES[fmt]
    fin = L  # expert input width (== d for the standard MoE)
    rows_tc = stats.get("tc_rows", 0)
    rows_st = stats.get("stream_rows", 0)
    e_tc = stats.get("tc_experts", 0)
    e_st = stats.get("stream_experts", 0)
    if phase == "expert_up_gemm":
        return 2.0 * rows_tc * fin * g * m, 2.0 * g * m * fin * e_tc
    if phase == "expert_down_gemm":
        return 2.0 * rows_tc * m * fin, 2.0 * fin * m * e_tc
    if phase == "expert_up_stream":
        return 2.0 * rows_st * fin * g * m, wb * g * m * fin * e_st
    if phase == "expert_down_stream":
        return 2.0 * rows_st * m * fin, wb * fin * m * e_st
    if phase == "router_proj_gemm":
        n_out = (L if cfg.has_proj else 0) + nt
        return 2.0 * T * d * n_out, 2.0 * (n_out * d + T * d)
    if phase == "up_proj_gemm":  # W_up and the residual x in, y out
        return 2.0 * T * L * d, 2.0 * (d * L + 2 * T * d)
    if phase == "shared_expert":
        ms = getattr(cfg, "shared_m", 0)
        return 2.0 * T * (g + 1) * d * ms, 2.0 * ((g + 1) * d * ms + T * (d + ms) + T * (ms + 2 * d))
    if phase == "combine":
        return 2.0 * T * cfg.top_k * L, 2.0 * (rows_tc + rows_st) * L + 2.0 * T * L
    if phase == "ep_regroup":  # three launches: counts, rows to expert-major order (read + write), and back
        return 0.0, 2.0 * 2 * 2 * (rows_tc + rows_st) * L / 3
    return 0.0, 0.0


def rooflines(cfg, stats, T, phases, peaks, step_ms):
    """The dominant kernel's roofline (from its phase time per launch) and the whole step's, plus the number of
    the library's kernel launches per step."""
    launches = sum(n for _, n in phases.values())
    dom = max(phases, key=lambda k: phases[k][0])
    dom_ms, dom_n = phases[dom]
    flops, nbytes = phase_units(cfg, stats, T, dom)
    per_launch_ms = dom_ms / max(dom_n, 1)
    intensity = flops / max(nbytes, 1.0)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    fmt = getattr(cfg, "expert_fmt", 0)
    rate = EXPERT_RATE[fmt] if dom.startswith("expert_") else 1.0
    if intensity >= ridge * rate:
        # a contraction takes the peak of its own dtype: block-scaled expert GEMMs run at the nominal
        # fp8 / fp4 : bf16 ratio times the measured bf16 peak
        roof = {"bound": "tensor", "achieved": flops / (per_launch_ms / 1e3) / 1e12,
                "peak": peaks["bf16_tflops"] * rate, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / (per_launch_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["launch_ms"] = per_launch_ms
    roof["algorithmic_per_launch"] = {"flops": flops, "bytes": nbytes}
    roof["traffic"] = NCU_TRAFFIC.get((cfg.name, dom))
    roof["peak_source"] = peaks["source"] + (" (burst)" if roof["bound"] == "tensor" else "") + (
        f", bf16 x {rate:g} (nominal ratio of the expert dtype)" if roof["bound"] == "tensor" and rate != 1.0 else "")

    F, B, F_eff = layer_work(cfg, stats, T)
    t_f, t_b = F_eff / (peaks["bf16_tflops"] * 1e12), B / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_f, t_b)
    layer_roof = {"flops": F, "bytes": B, "t_roof_us": t_roof * 1e6, "t_step_us": step_ms * 1e3,
                  "frac": t_roof / (step_ms / 1e3), "bound": "tensor" if t_f >= t_b else "hbm"}
    return roof, layer_roof, launches


# ----------------------------------------------------------------------------- GPU arm
def setup_layer(cfg, rank, device):
    layer = synth.make_layer(cfg)
    xs = [synth.make_tokens(cfg, cfg.tokens, seed=1000 * (rank + 1) + i) for i in range(N_INPUT_BATCHES)]
    return layer, xs


def run_gpu(cfg, steps, warmup, rank, world, device, peaks, with_e2e=True, with_clocks=True, grouped_kind=None):
    torch.cuda.set_device(device)
    layer, xs = setup_layer(cfg, rank, device)
    T = cfg.tokens
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=T, device=f"cuda:{device}")
    if grouped_kind is not None:
        lmoe.lmoe_set_grouped_gemm(mod.h, grouped_kind)
    xd = [x.to(f"cuda:{device}") for x in xs]
    yd = torch.empty_like(xd[0])
    stream = torch.cuda.current_stream()

    # routing statistics averaged over the input batches (path split for the per-kernel work)
    acc = {}
    for xb in xd:
        mod.forward(xb, yd)
        torch.cuda.synchronize()
        st = lmoe.lmoe_routing_stats(mod.h)
        for k, v in st.items():
            acc[k] = acc.get(k, 0) + v / len(xd)
    stats = acc

    dev = torch.device(f"cuda:{device}")
    barrier = lambda: dist_barrier(world)  # noqa: E731
    max_over_ranks = lambda v: dist_max(v, world, dev)  # noqa: E731

    for i in range(warmup):
        mod.forward(xd[i % N_INPUT_BATCHES], yd)
    torch.cuda.synchronize()
    status = mod.last_error()
    if status != 0:
        raise RuntimeError(f"device error during warm-up: {lmoe.lmoe_status_string(status)}")

    # ---------------------------------------------------------------- device-timed region (the headline)
    # No per-phase events here: an event between two kernels costs ~2 us of GPU time and breaks the
    # programmatic overlap of the launches, which slows a ~0.3 ms decode step by ~15%.
    clocks = ClockSampler(_smi_id(device)) if with_clocks else None
    if clocks:
        clocks.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        mod.forward(xd[i % N_INPUT_BATCHES], yd)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop() if clocks else None
    status = mod.last_error()
    if status != 0:
        raise RuntimeError(f"device error in the timed region: {lmoe.lmoe_status_string(status)}")
    ms_max = max_over_ranks(ms)

    # ---------------------------------------------------------------- kernel-timed region (the roofline)
    # The same steps again with CUDA events around every phase, on the stream the kernels run on.
    lmoe.lmoe_set_profiling(mod.h, True, steps)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        mod.forward(xd[i % N_INPUT_BATCHES], yd)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_profiled = ev0.elapsed_time(ev1)
    phases = lmoe.lmoe_phase_times(mod.h)
    lmoe.lmoe_set_profiling(mod.h, False)
    status = mod.last_error()
    if status != 0:
        raise RuntimeError(f"device error in the kernel-timed region: {lmoe.lmoe_status_string(status)}")

    # ---------------------------------------------------------------- the same steps replayed from CUDA graphs
    # one graph per input batch, each holding one whole forward (its launches and the shared expert's stream)
    graph = None
    if with_e2e:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            mod.forward(xd[0], yd)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graphs = []
        for i in range(N_INPUT_BATCHES):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                mod.forward(xd[i], yd)
            graphs.append(gr)
        for i in range(warmup):
            graphs[i % N_INPUT_BATCHES].replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(steps):
            graphs[i % N_INPUT_BATCHES].replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        g_ms = max_over_ranks(ev0.elapsed_time(ev1))
        status = mod.last_error()
        if status != 0:
            raise RuntimeError(f"device error in the graph-replay region: {lmoe.lmoe_status_string(status)}")
        graph = {"value": world * T * steps / (g_ms / 1e3), "unit": "tokens/s", "ms_per_step": g_ms / steps,
                 "launch": "one CUDA graph per forward, replayed"}
        del graphs

    # ---------------------------------------------------------------- end to end through host buffers
    e2e = None
    if with_e2e:
        xh = [x.pin_memory() for x in xs]
        yh = torch.empty_like(xh[0]).pin_memory()
        for i in range(warmup):
            mod.forward_host(xh[i % N_INPUT_BATCHES], yh)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(steps):
            mod.forward_host(xh[i % N_INPUT_BATCHES], yh)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1))
        e2e = {"value": world * T * steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(xh[0].numel() * xh[0].element_size()),
               "d2h_bytes_per_step": int(yh.numel() * yh.element_size()), "ms_per_step": e2e_ms / steps}

    roof, layer_roof, launches = rooflines(cfg, stats, T, phases, peaks, ms_max / steps)
    mod.close()
    roof["kernel_timed_ms_per_step"] = ms_profiled / steps
    return {"ms": ms_max, "phases": phases, "launches": launches, "roofline": roof, "layer_roofline": layer_roof,
            "e2e": e2e, "clocks": clk, "stats": stats, "graph": graph}


def run_ep(cfg, steps, warmup, rank, world, device, peaks, exchange_mode="auto"):
    """Expert-parallel steps: this rank holds n_ffn / world experts and routes its own tokens.

    Rows cross ranks by NCCL all-to-all; with one rank nothing moves. Decode-size batches take the block
    exchange (equal blocks per rank pair, no host wait); larger ones the packed exchange, whose step includes
    one host wait (the counts that size it).
    """
    from latent_mixture_experts_gemm_b200 import expert_parallel as xp
    torch.cuda.set_device(device)
    layer, xs = setup_layer(cfg, rank, device)
    T = cfg.tokens
    limit = {"auto": 64 << 20, "packed": -1, "blocks": 1 << 62}[exchange_mode]
    rk = xp.ExpertParallelLatentMoE(cfg, layer, max_tokens=T, ep_size=world, ep_rank=rank, device=f"cuda:{device}",
                                    block_limit_bytes=limit)
    xd = [x.to(f"cuda:{device}") for x in xs]
    yd = torch.empty_like(xd[0])
    stream = torch.cuda.current_stream()
    dev = torch.device(f"cuda:{device}")
    barrier = lambda: dist_barrier(world)  # noqa: E731
    max_over_ranks = lambda v: dist_max(v, world, dev)  # noqa: E731

    def check(where):
        status = rk.last_error()
        if status != 0:
            raise RuntimeError(f"device error {where}: {lmoe.lmoe_status_string(status)}")

    # expert-side routing statistics (rows this rank's experts received) and the rows sent to other ranks
    acc, sent_away = {}, 0.0
    nl = cfg.n_ffn // world
    for xb in xd:
        rk.forward(xb, yd)
        torch.cuda.synchronize()
        for k, v in lmoe.lmoe_routing_stats(rk.mod.h).items():
            acc[k] = acc.get(k, 0) + v / len(xd)
        sc = rk.send_counts.cpu().view(world, nl).sum(1)
        sent_away += float(sc.sum() - sc[rank]) / len(xd)
    stats = acc
    for i in range(warmup):
        rk.forward(xd[i % N_INPUT_BATCHES], yd)
    torch.cuda.synchronize()
    check("during warm-up")

    clocks = ClockSampler(_smi_id(device))
    clocks.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        rk.forward(xd[i % N_INPUT_BATCHES], yd)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    check("in the timed region")
    ms_max = max_over_ranks(ms)

    lmoe.lmoe_set_profiling(rk.mod.h, True, steps)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        rk.forward(xd[i % N_INPUT_BATCHES], yd)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_profiled = ev0.elapsed_time(ev1)
    phases = lmoe.lmoe_phase_times(rk.mod.h)
    lmoe.lmoe_set_profiling(rk.mod.h, False)
    check("in the kernel-timed region")

    # end to end: pinned host tokens in, host output back, every step
    xh = [x.pin_memory() for x in xs]
    yh = torch.empty_like(xh[0]).pin_memory()
    xin = torch.empty_like(xd[0])

    def host_step(i):
        xin.copy_(xh[i % N_INPUT_BATCHES], non_blocking=True)
        rk.forward(xin, yd)
        yh.copy_(yd, non_blocking=True)

    for i in range(warmup):
        host_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        host_step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1))
    check("in the end-to-end region")
    e2e = {"value": world * T * steps / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(xh[0].numel() * xh[0].element_size()),
           "d2h_bytes_per_step": int(yh.numel() * yh.element_size()), "ms_per_step": e2e_ms / steps}

    # With the block exchange a step has no host wait, so one rank's step can be captured in a CUDA graph and
    # replayed (with several ranks the graph would hold the NCCL exchanges: not measured here).
    graph = None
    if rk.block_exchange and world == 1:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            rk.forward(xd[0], yd)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graphs = []
        for i in range(N_INPUT_BATCHES):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                rk.forward(xd[i], yd)
            graphs.append(gr)
        for i in range(warmup):
            graphs[i % N_INPUT_BATCHES].replay()
        torch.cuda.synchronize()
        ev0.record(stream)
        for i in range(steps):
            graphs[i % N_INPUT_BATCHES].replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        g_ms = ev0.elapsed_time(ev1)
        check("in the graph-replay region")
        graph = {"value": T * steps / (g_ms / 1e3), "unit": "tokens/s", "ms_per_step": g_ms / steps,
                 "launch": "one CUDA graph per expert-parallel step (block exchange, one rank), replayed"}
        del graphs

    roof, layer_roof, launches = rooflines(cfg, stats, T, phases, peaks, ms_max / steps)
    roof["kernel_timed_ms_per_step"] = ms_profiled / steps
    blocks = rk.block_exchange
    moved = (2 * 2 * (world - 1) * rk.block_rows * cfg.latent) if blocks else 2 * 2 * sent_away * cfg.latent
    exchange = {"ranks": world, "rows_sent_to_other_ranks_per_step": sent_away,
                "bytes_over_nvlink_per_step": moved,
                "mode": (f"blocks of {rk.block_rows} rows per rank pair, equal splits: no count read on the host"
                         if blocks else "packed rows, split sizes from the counts read on the host"),
                "collective": ("NCCL all_to_all_single (counts, row blocks, row blocks back)" if blocks else
                               "NCCL all_to_all_single (counts, rows, rows back)") if world > 1 else "none (one rank)"}
    rk.close()
    return {"ms": ms_max, "phases": phases, "launches": launches, "roofline": roof, "layer_roofline": layer_roof,
            "e2e": e2e, "clocks": clk, "stats": stats, "exchange": exchange, "graph": graph}


# ----------------------------------------------------------------------------- oracle (CPU) arm
def oracle_rate(cfg, layer, budget_s: float):
    """Tokens/s of the fp64 oracle on a bounded sample of the workload: the first n tokens, n chosen from a
    one-token probe so one pass takes about `budget_s`; a workload smaller than that is passed over whole,
    repeatedly, until the budget is spent."""
    import oracle
    t0 = time.perf_counter()
    oracle.forward(cfg, layer, x=layer["x"][:1], want=("y",))
    one = max(time.perf_counter() - t0, 1e-4)
    n = int(max(1, min(cfg.tokens, budget_s / one * oracle.num_threads() * 0.8)))
    passes, tokens, t0 = 0, 0, time.perf_counter()
    while True:
        oracle.forward(cfg, layer, x=layer["x"][:n], want=("y",))
        passes += 1
        tokens += n
        dt = time.perf_counter() - t0
        if dt >= 0.5 * budget_s or passes >= 200:
            break
    return tokens / dt, n, passes, dt, oracle.num_threads()


def cpu_baseline(cfg, budget_s=15.0):
    layer = synth.make_layer(cfg)
    rate, n, passes, dt, cores = oracle_rate(cfg, layer, budget_s)
    return {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} pass(es) over {n} of the {cfg.tokens} tokens of {cfg.name}, fp64, {dt:.1f} s"}


def run_reference(args, cfg, rank, world):
    """The fp64 oracle as it stands, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    layer = synth.make_layer(cfg)
    total_budget = 150.0
    t0 = time.perf_counter()
    oracle.forward(cfg, layer, x=layer["x"][:1], want=("y",))
    one = max(time.perf_counter() - t0, 1e-4)
    per_step = total_budget / max(args.steps + args.warmup, 1)
    n = int(max(1, min(cfg.tokens, per_step / one * oracle.num_threads() * 0.8)))
    for _ in range(args.warmup):
        oracle.forward(cfg, layer, x=layer["x"][:n], want=("y",))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(cfg, layer, x=layer["x"][:n], want=("y",))
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{n} of the {cfg.tokens} tokens of {cfg.name} per step, fp64"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


EXPERT_FORMATS = ["bf16", "mxfp8 (e4m3 weights and expert inputs)", "mxfp4 (e2m1 weights, mxfp8 expert inputs)",
                  "nvfp4 (e2m1 weights and expert inputs, e4m3 scale per 16, fp32 scale per expert matrix)"]


def compute_dtype(cfg):
    """The arithmetic types the path computes in: bf16 tensor-core GEMMs, plus block-scaled expert GEMMs."""
    return ["bf16", "bf16+mxfp8", "bf16+mxfp4/mxfp8", "bf16+nvfp4"][cfg.expert_fmt]


def workload_config(cfg):
    return {"workload": cfg.name, "tokens": cfg.tokens, "d": cfg.d, "latent": cfg.latent, "m": cfg.m,
            "experts": cfg.n_ffn, "bypass_experts": [cfg.n_zero, cfg.n_copy, cfg.n_const], "top_k": cfg.top_k,
            "shared_expert_width": cfg.shared_m,
            "expert_format": EXPERT_FORMATS[cfg.expert_fmt],
            "act": ["relu2", "swiglu", "identity"][cfg.act], "projection": bool(cfg.has_proj),
            "l2": "inputs larger than L2 (the touched expert weights, read every step, exceed the 126 MB L2)",
            "parallelism": "replicas (tokens shard with no exchange)"}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, help="override the workload's token count (profiling runs)")
    ap.add_argument("--impl", default="lmoe", choices=["lmoe", "reference"])
    ap.add_argument("--no-secondary", action="store_true", help="skip the other workloads' measurements")
    ap.add_argument("--secondary", default=",".join(SECONDARY_WORKLOADS),
                    help="comma-separated workloads measured beside the main one (reported under `secondary`)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ep", action="store_true", help="expert parallelism over the ranks instead of replicas")
    ap.add_argument("--ep-exchange", default="auto", choices=["auto", "packed", "blocks"],
                    help="--ep: the block exchange for small batches (auto), or one of the two always")
    ap.add_argument("--grouped-kind", type=int, choices=[0, 1], default=None,
                    help="kernel of the grouped expert GEMMs (lmoe_set_grouped_gemm) for the main workload")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = synth.WORKLOADS[args.workload]
    if args.tokens:
        cfg = cfg.with_(tokens=args.tokens, name=f"{cfg.name}_T{args.tokens}")

    if args.impl == "reference":
        line = run_reference(args, cfg, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime

        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device(f"cuda:{local}"))
    peaks = load_peaks()
    try:
        if args.ep:
            res = run_ep(cfg, args.steps, args.warmup, rank, world, local, peaks, args.ep_exchange)
        else:
            res = run_gpu(cfg, args.steps, args.warmup, rank, world, local, peaks, grouped_kind=args.grouped_kind)
        secondary = None
        if not args.ep and not args.no_secondary:
            secondary = []
            for name in [w for w in args.secondary.split(",") if w and w != args.workload]:
                sc = synth.WORKLOADS[name]
                # decode batches take well under a millisecond each: at least 100 timed steps, so that the
                # clock sampler sees the region and a single slow step moves the mean little
                s_steps = max(100, min(args.steps, 400)) if sc.tokens <= 32 else max(3, min(args.steps, 20))
                r2 = run_gpu(sc, s_steps, args.warmup, rank, world, local, peaks, with_e2e=False)
                secondary.append({"workload": sc.name, "config": workload_config(sc), "dtype": compute_dtype(sc),
                                  "steps": s_steps,
                                  "tokens_per_s": world * sc.tokens * s_steps / (r2["ms"] / 1e3),
                                  "ms_per_step": r2["ms"] / s_steps, "roofline": r2["roofline"],
                                  "layer_roofline": r2["layer_roofline"], "clocks": r2["clocks"],
                                  "phases_ms_per_step": {k: v[0] / s_steps for k, v in r2["phases"].items()},
                                  "gpu_launches": r2["launches"], "routing": r2["stats"]})
    finally:
        pass
    if rank == 0:
        T = cfg.tokens
        value = world * T * args.steps / (res["ms"] / 1e3)
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["ms"] / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": compute_dtype(cfg), "data": "synthetic",
                "config": workload_config(cfg), "roofline": res["roofline"],
                "layer_roofline": res["layer_roofline"], "e2e": res["e2e"], "gpu_launches": res["launches"],
                "clocks": res["clocks"],
                "phases_ms_per_step": {k: v[0] / args.steps for k, v in res["phases"].items()},
                "routing": res["stats"]}
        if args.grouped_kind is not None:
            line["config"]["grouped_gemm_kind"] = args.grouped_kind
        if res.get("graph") is not None:
            line["graph_replay"] = res["graph"]
        if secondary is not None:
            line["secondary"] = secondary
        if args.ep:
            line["config"]["parallelism"] = (f"ep{world}: each rank holds {cfg.n_ffn // world} of the {cfg.n_ffn} "
                                             "FFN experts and routes its own tokens")
            line["exchange"] = res["exchange"]
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(cfg)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
