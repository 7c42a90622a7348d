#!/usr/bin/env python
"""Throughput of one K2-style MoE FFN layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload k2_decode|k2_prefill|k2_skew|v3|tiny]

One step = one full layer forward (route, permute, grouped SwiGLU experts with
the shared expert, combine) over one batch of T synthetic tokens, inputs and
weights resident in HBM.  Prints ONE JSON line on rank 0.

  ours       the CUDA library through its C ABI (moe_layer_forward)
  reference  the fp64 CPU oracle on the host cores, on a bounded token sample
             of the same workload (rows are independent, so tokens/s of a
             sample is the oracle's rate on the workload)

With N > 1 (torchrun, one process per GPU) every rank runs its own replica on
its own batch (weak scaling; the layer has no exchange step on one GPU per
replica); the time is the max over ranks and value counts all ranks' tokens.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "K2 MoE-layer tokens/s; % of HBM (decode) / bf16 tensor (prefill) roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# timed steps per workload: the device-timed region stays near a second (for
# the clock samples) and the oracle reference arm (about a second per step on
# a K2 token) within a few minutes
DEFAULT_STEPS = {"k2_decode": 150, "tiny": 200, "v3": 100, "k2_skew": 100, "k2_prefill": 60}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="k2_decode")
    p.add_argument("--balance", type=int, default=0, metavar="S",
                   help="time the load-balancing pass instead of the layer: router scores, "
                        "route, permute, the sequence-level loss over sequences of S tokens "
                        "and the bias update")
    p.add_argument("--weights", choices=["bf16", "fp8", "w8a8", "w4a16"], default="bf16",
                   help="expert weights: bf16; fp8 = routed experts stored as E4M3 codes with "
                        "one power-of-two scale per 128x128 block, bf16 compute; w4a16 = routed "
                        "experts as INT4 with a bf16 scale per group of 32, bf16 compute; w8a8 = FP8 "
                        "compute in every expert, E4M3 weights and activations with one "
                        "power-of-two scale per row (weights quantized once, untimed)")
    p.add_argument("--cpu-sample", type=int, default=None,
                   help="tokens in the oracle's timed sample (default: sized from the core count)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="time the decode headline only (the default run also times k2_prefill, "
                        "k2_skew and v3 on the same weights)")
    p.add_argument("--pdl-ab", action="store_true",
                   help="instead of the bench line: time the layer with programmatic dependent "
                        "launch off and on, alternating (4 rounds of 50 calls each), and print "
                        "the medians")
    p.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                   help="override a workload field (T, d, E, k, inter), e.g. a small case of\n"
                        "the same kernels for profiling: --set E=16")
    a = p.parse_args(argv)
    if a.steps is None:
        a.steps = DEFAULT_STEPS.get(a.workload, 100)
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    return a


# ------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the timed region
    runs: NVML polled every 2 ms from a thread (so a 20-step decode run of about
    70 ms still gets dozens of samples), else nvidia-smi's loop mode.  Reads only;
    no setting of the GPU is changed."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    # NVML clock-event reason bits of the four names above
    NVML_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                 "sw_power_cap": 0x4}
    PERIOD_S = 0.002
    PERIOD_MS = 20          # nvidia-smi fallback

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.samples = []       # (time, sm MHz, reasons set), NVML
        self.smax = None
        self._stop = threading.Event()
        self.thread = None

    def _nvml_handle(self):
        try:
            import pynvml
            pynvml.nvmlInit()
        except Exception:
            return None
        self._nvml = pynvml
        try:
            # the GPU this process uses, by PCI address (NVML counts GPUs physically)
            import torch
            pr = torch.cuda.get_device_properties(self.gpu)
            bus = "%08X:%02X:%02X.0" % (getattr(pr, "pci_domain_id"), getattr(pr, "pci_bus_id"),
                                        getattr(pr, "pci_device_id"))
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            pass
        try:
            return pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        except Exception:
            return None

    def _poll_nvml(self, h):
        nv = self._nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self._stop.is_set():
            try:
                t = time.time()
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = get_reasons(h) if get_reasons else 0
                self.samples.append((t, float(sm), {n for n, b in self.NVML_BITS.items() if bits & b}))
            except Exception:
                return
            time.sleep(self.PERIOD_S)

    def __enter__(self):
        h = self._nvml_handle()
        if h is not None:
            try:
                self.smax = float(self._nvml.nvmlDeviceGetMaxClockInfo(h, self._nvml.NVML_CLOCK_SM))
            except Exception:
                self.smax = None
            self.thread = threading.Thread(target=self._poll_nvml, args=(h,), daemon=True)
            self.thread.start()
            time.sleep(0.05)
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        return time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        else:
            self._stop.set()
            if self.thread is not None:
                self.thread.join(timeout=1.0)
        return False

    def summary(self, t0, t1):
        sm, smax, reasons = [], self.smax, set()
        for ts, mhz, rs in self.samples:
            if t0 <= ts <= t1:
                sm.append(mhz)
                reasons |= rs
        for ts, line in self.lines:
            if not (t0 <= ts <= t1):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        src = "nvml" if self.samples else "nvidia-smi"
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": 0,
                    "source": src}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "source": src}


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = ["sparse_moe_ffn_sigmoid_b200/csrc/gemm.cuh", "sparse_moe_ffn_sigmoid_b200/csrc/ptx.cuh",
                  "sparse_moe_ffn_sigmoid_b200/csrc/common.cuh",
                  "sparse_moe_ffn_sigmoid_b200/csrc/quant.cuh",
                  "sparse_moe_ffn_sigmoid_b200/csrc/gemv.cuh"]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if the
    kernel sources are unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(KERNEL_SOURCES)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and parts[0] == workload and parts[1] == kernel and \
                    parts[3] == digest:
                return float(parts[2])
    return None


# ----------------------------------------------------------- multi-rank

def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest per-rank value over all ranks (the slowest rank's time)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms_total: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_total / 1e3)


# ----------------------------------------------------- accounting (per step)

def layer_accounting(cfg, touched: int, weights: str = "bf16"):
    """Algorithmic bytes and FLOPs of one layer forward, and of its two GEMMs.

    touched: routed experts with at least one token this step (the shared
    expert is always touched on top).  Weight bytes per expert follow the
    pages' 3 x d x inter parameter count ("Kimi K2.5 Q&A", Q2.1).  With FP8
    storage a routed expert's weights are one byte each plus one int8 scale
    per 128 x 128 block; the shared expert stays bf16.  With FP8 compute every
    expert's weights (shared too) are one byte each plus one int8 exponent per
    row, and the GEMMs read their token rows as one byte per element plus one
    exponent per row."""
    T, d, E, k, I = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter
    rows = T * (k + 1)
    w_gu = 2 * I * d * 2                 # gate + up weights of one expert, bytes
    w_dn = d * I * 2
    a_in_gu, a_in_dn = rows * d * 2, rows * I * 2      # token rows the GEMMs read
    if weights == "fp8":
        r_gu = 2 * I * d + (2 * I // 128) * (d // 128)
        r_dn = d * I + (d // 128) * (I // 128)
    elif weights == "w4a16":
        r_gu = I * d + (2 * I) * (d // 32) * 2
        r_dn = d * I // 2 + d * (I // 32) * 2
    elif weights == "w8a8":
        r_gu, r_dn = 2 * I * d + 2 * I, d * I + d
        w_gu, w_dn = r_gu, r_dn
        a_in_gu, a_in_dn = rows * (d + 1), rows * (I + 1)
    else:
        r_gu, r_dn = w_gu, w_dn
    acc = {}
    acc["gate_up_bytes"] = touched * r_gu + w_gu + a_in_gu + rows * I * 2
    acc["down_bytes"] = touched * r_dn + w_dn + a_in_dn + rows * d * 2
    acc["gate_up_flops"] = 2.0 * rows * 2 * I * d
    acc["down_flops"] = 2.0 * rows * I * d
    acc["router_flops"] = 2.0 * T * d * E
    acc["weight_bytes"] = touched * (r_gu + r_dn) + (w_gu + w_dn) + E * d * 2
    acc["flops"] = acc["gate_up_flops"] + acc["down_flops"] + acc["router_flops"]
    return acc


# ------------------------------------------------ other full-size workloads

# Timed after the decode line in the default run, on the decode run's weights.
EXTRA_WORKLOADS = ("k2_prefill", "k2_skew", "v3")
EXTRA_TIMED_MS = 1000.0     # device time each one's timed region aims at (clock samples)


def extra_inputs(name, g, dev, seed):
    """Inputs of another full-size workload on the decode run's weight set.
    The expert shapes are the same (d = 7168, inter = 2048), so the 384 routed
    experts, the router rows and the shared expert are reused (the first 256
    experts and router rows for the DeepSeek-V3 shape); x and the selection
    bias are drawn for the workload with the distributions moe_inputs states."""
    import torch
    from moe_inputs import CONFIGS, make_bias
    cfg = CONFIGS[name]
    E = cfg.E
    if cfg.d != g["x"].shape[1] or cfg.inter != g["w_down"].shape[2] or E > g["w_router"].shape[0]:
        raise ValueError(f"{name}: expert shapes differ from the decode weight set")
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    x = torch.randn((cfg.T, cfg.d), generator=gen, device=dev, dtype=torch.float32)
    inp = dict(x=x.to(torch.bfloat16), w_router=g["w_router"][:E], bias=make_bias(cfg, gen, dev),
               w_gate_up=g["w_gate_up"][:E], w_down=g["w_down"][:E], ws_gate_up=g["ws_gate_up"],
               ws_down=g["ws_down"])
    return cfg, inp


def touched_experts(moe, cfg, g, dev) -> int:
    """Routed experts with at least one token in this batch (our own route and
    permute kernels)."""
    import torch
    T, d, E, k, I = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter
    ws = torch.empty(moe.moe_workspace_size(T, d, E, k, I), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    moe.moe_route(g["x"], g["w_router"], g["bias"], k, cfg.scale, idx, w, ws)
    i32 = lambda n: torch.empty((n,), dtype=torch.int32, device=dev)
    counts, offs, rtok, srow = i32(E), i32(E + 1), i32(T * k), i32(T * k)
    moe.moe_permute(idx, E, counts, offs, rtok, srow, ws)
    return int((counts > 0).sum().item())


def time_extra_workload(moe, cfg, inp, dev, warmup, peaks, peak_src, gpu_index):
    """One bf16 layer workload, device-timed like the headline (CUDA events on
    the launching stream, inputs resident, clocks sampled during the timed
    region), with its tensor fraction against both measured bf16 peaks, its
    HBM fraction, and its time in SM cycles at the sampled clock."""
    import torch
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        moe.moe_layer_forward(inp["x"], inp["w_router"], inp["bias"], inp["w_gate_up"],
                              inp["w_down"], inp["ws_gate_up"], inp["ws_down"], k, cfg.scale, out)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(warmup):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    ms_warm = start.elapsed_time(end) / warmup
    steps = int(min(400, max(20, math.ceil(EXTRA_TIMED_MS / max(ms_warm, 1e-3)))))
    touched = touched_experts(moe, cfg, inp, dev)

    moe.moe_profile_begin(steps)
    with ClockSampler(gpu_index) as clk:
        torch.cuda.synchronize(dev)
        t0 = clk.mark()
        start.record(stream)
        for _ in range(steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        t1 = clk.mark()
    ms = start.elapsed_time(end) / steps
    n_calls, kernel_ms = moe.moe_profile_end()
    if moe.moe_device_status() != 0:
        raise SystemExit(f"{cfg.name}: device status not clean after the timed region")
    clocks = clk.summary(t0, t1)

    acc = layer_accounting(cfg, touched)
    burst = peaks["bf16_tflops"]
    sust = peaks.get("bf16_tflops_sustained", burst)
    hbm_peak = peaks["hbm_gbs"]
    tflops = acc["flops"] / (ms / 1e3) / 1e12
    gu_ms = kernel_ms.get("gemm_gate_up_swiglu", 0.0) / max(n_calls, 1)
    gu_tflops = acc["gate_up_flops"] / (gu_ms / 1e3) / 1e12 if gu_ms > 0 else None
    hbm = acc["weight_bytes"] / (ms / 1e3) / 1e9
    mhz = clocks["sm_mhz"]
    return {
        "T": T, "E": E, "k": k, "scale": cfg.scale, "bias": cfg.bias, "steps": steps,
        "warmup": warmup, "ms_per_step": ms, "tokens_per_s": T / (ms / 1e3),
        "touched_experts": touched, "flops": acc["flops"], "weight_bytes": acc["weight_bytes"],
        "tensor": {"achieved_tflops": tflops, "frac_of_burst": tflops / burst,
                   "frac_of_sustained": tflops / sust, "peak_burst_tflops": burst,
                   "peak_sustained_tflops": sust, "peak_source": f"{peak_src} bf16_tflops / "
                                                                 "bf16_tflops_sustained"},
        "gate_up_kernel": {"avg_launch_ms": gu_ms, "achieved_tflops": gu_tflops,
                           "frac_of_burst": gu_tflops / burst if gu_tflops else None,
                           "frac_of_sustained": gu_tflops / sust if gu_tflops else None},
        "hbm": {"achieved_gbs": hbm, "frac": hbm / hbm_peak, "peak_gbs": hbm_peak,
                "peak_source": f"{peak_src} hbm_gbs"},
        "ideal_ms": {"tensor_burst": acc["flops"] / (burst * 1e12) * 1e3,
                     "tensor_sustained": acc["flops"] / (sust * 1e12) * 1e3,
                     "hbm": acc["weight_bytes"] / (hbm_peak * 1e9) * 1e3},
        # the attainable bound: the slower of the weight stream and the tensor
        # time at the burst peak, and the step's fraction of it
        "attainable": {"ms": max(acc["weight_bytes"] / (hbm_peak * 1e9),
                                 acc["flops"] / (burst * 1e12)) * 1e3,
                       "bound": "hbm" if acc["weight_bytes"] / (hbm_peak * 1e9) >=
                                acc["flops"] / (burst * 1e12) else "tensor",
                       "frac": max(acc["weight_bytes"] / (hbm_peak * 1e9),
                                   acc["flops"] / (burst * 1e12)) * 1e3 / ms},
        "clocks": clocks,
        # ms x median SM MHz / 1000: the step in millions of SM cycles, so that a
        # power-capped clock shows as a lower MHz at an unchanged cycle count
        "sm_mcycles_per_step": ms * mhz / 1e3 if mhz else None,
        "kernel_ms_per_step": {kk: v / max(n_calls, 1) for kk, v in kernel_ms.items()},
    }


# ------------------------------------------------------------------- oracle

class OracleSample:
    """A fixed, evenly spaced token sample of the workload with everything the
    oracle needs copied to the host once (x rows, router, the experts those
    tokens select, the shared expert).  Rows are independent, so the oracle's
    tokens/s on the sample is its rate on the workload."""

    def __init__(self, cfg, inputs_dev, n_tokens, weights: str = "bf16"):
        import torch
        import oracle
        self.cfg = cfg
        T = cfg.T
        n = max(1, min(n_tokens, T))
        self.tokens = sorted(set(int(round(i * (T - 1) / max(n - 1, 1))) for i in range(n)))
        sel = torch.tensor(self.tokens, device=inputs_dev["x"].device)
        self.x = inputs_dev["x"].index_select(0, sel).cpu()
        self.wr = inputs_dev["w_router"].cpu()
        self.bias = inputs_dev["bias"].cpu()
        self.threads = min(host_cores(), len(self.tokens))
        # routing of a row depends on that row only
        ridx, _, _ = oracle.route(self.x, self.wr, self.bias, cfg.k, cfg.scale, nthreads=self.threads)
        self.need = sorted(set(ridx.reshape(-1).tolist()))
        self.egu = [None] * cfg.E
        self.edn = [None] * cfg.E
        self.weights = weights
        for e in self.need:
            self.egu[e] = inputs_dev["w_gate_up"][e].cpu()
            self.edn[e] = inputs_dev["w_down"][e].cpu()
            if weights == "fp8":
                # the weights FP8 storage stands for, from the oracle's own quantizer
                self.egu[e] = oracle.dequantize_fp8(*oracle.quantize_fp8(self.egu[e]))
                self.edn[e] = oracle.dequantize_fp8(*oracle.quantize_fp8(self.edn[e]))
            elif weights == "w4a16":
                self.egu[e] = oracle.dequantize_int4(*oracle.quantize_int4(self.egu[e]))
                self.edn[e] = oracle.dequantize_int4(*oracle.quantize_int4(self.edn[e]))
        self.sgu, self.sdn = inputs_dev["ws_gate_up"].cpu(), inputs_dev["ws_down"].cpu()
        if weights == "w8a8":
            # FP8-compute weights from the oracle's own row quantizer
            host = {"w_gate_up": self.egu, "w_down": self.edn, "ws_gate_up": self.sgu,
                    "ws_down": self.sdn}
            qe, self.qs = oracle.quantize_expert_rows(host, self.need)
            self.qe = [qe.get(e) for e in range(cfg.E)]

    def run(self) -> float:
        """Seconds for the oracle's full layer (routing + experts) on the sample."""
        import oracle
        t0 = time.perf_counter()
        ridx, rw, _ = oracle.route(self.x, self.wr, self.bias, self.cfg.k, self.cfg.scale,
                                   nthreads=self.threads)
        if self.weights == "w8a8":
            oracle.moe_rows_fp8(self.x, ridx, rw, self.qe, self.qs, nthreads=self.threads)
        else:
            oracle.moe_rows(self.x, ridx, rw, self.egu, self.edn, self.sgu, self.sdn,
                            nthreads=self.threads)
        return time.perf_counter() - t0

    def describe(self) -> str:
        fp8 = {"fp8": " (routed weights: the oracle's FP8 quantization, dequantized)",
               "w4a16": " (routed weights: the oracle's INT4 quantization, dequantized)",
               "w8a8": " (FP8 compute: the oracle's per-row E4M3 quantization of weights "
                       "and activations)"}.get(self.weights, "")
        return (f"{len(self.tokens)} of {self.cfg.T} tokens (evenly spaced), full routing + "
                f"{len(self.need)} routed experts + shared expert, fp64{fp8}")


def default_cpu_sample(cfg, weights: str = "bf16"):
    # ~0.8 GFLOP of fp64 per K2 token, one thread per token: 64 tokens keep a
    # 16-core host busy for several seconds without copying every expert.
    # With FP8 weights the oracle first quantizes every expert the sample
    # selects (about a second each), so the sample is smaller.
    if weights in ("fp8", "w8a8", "w4a16"):
        return min(cfg.T, 8)
    return min(cfg.T, max(64, 4 * host_cores()))


# --------------------------------------------------------------------- main

def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    from moe_inputs import CONFIGS, make_inputs
    if args.workload not in CONFIGS:
        raise SystemExit(f"unknown workload {args.workload}; choose from {sorted(CONFIGS)}")
    cfg = CONFIGS[args.workload]
    if args.set:
        fields = cfg.as_dict()
        for item in args.set:
            key, _, val = item.partition("=")
            if key not in ("T", "d", "E", "k", "inter"):
                raise SystemExit(f"--set: unknown field {key!r}")
            fields[key] = int(val)
        cfg = cfg.__class__(**fields)

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, cfg, world)
    if args.balance:
        return run_balance(args, cfg)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    import sparse_moe_ffn_sigmoid_b200 as moe

    dev = torch.device("cuda", local_rank)
    g = make_inputs(cfg, seed=rank, device=dev)
    T, d, E, k, I = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    fp8 = args.weights == "fp8"
    w8a8 = args.weights == "w8a8"
    w4 = args.weights == "w4a16"
    if w4:
        qgu, sgu = moe.moe_quantize_int4(g["w_gate_up"])
        qdn, sdn = moe.moe_quantize_int4(g["w_down"])
        torch.cuda.synchronize(dev)
    if fp8:
        # storage format conversion, once, outside every timed region
        qgu, egu = moe.moe_quantize_fp8(g["w_gate_up"])
        qdn, edn = moe.moe_quantize_fp8(g["w_down"])
        torch.cuda.synchronize(dev)
    if w8a8:
        wq = []
        for key in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
            wq += list(moe.moe_quantize_fp8_rows(g[key]))
        torch.cuda.synchronize(dev)

    def layer(x_in):
        if w4:
            moe.moe_layer_forward_w4a16(x_in, g["w_router"], g["bias"], qgu, sgu, qdn, sdn,
                                        g["ws_gate_up"], g["ws_down"], k, cfg.scale, out)
        elif w8a8:
            moe.moe_layer_forward_w8a8(x_in, g["w_router"], g["bias"], *wq, k, cfg.scale, out)
        elif fp8:
            moe.moe_layer_forward_fp8(x_in, g["w_router"], g["bias"], qgu, egu, qdn, edn,
                                      g["ws_gate_up"], g["ws_down"], k, cfg.scale, out)
        else:
            moe.moe_layer_forward(x_in, g["w_router"], g["bias"], g["w_gate_up"], g["w_down"],
                                  g["ws_gate_up"], g["ws_down"], k, cfg.scale, out)

    def step():
        layer(g["x"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if moe.moe_device_status() != 0:
        raise SystemExit("device status not clean after warm-up")
    launches_per_step = moe.moe_last_launch_count()
    if args.pdl_ab:
        if world > 1:
            raise SystemExit("--pdl-ab runs on one GPU")
        return run_pdl_ab(moe, args, cfg, step, stream, dev)

    touched = touched_experts(moe, cfg, g, dev)

    # ---------------------------------------------------------- timed region
    moe.moe_profile_begin(args.steps)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t_wall0 = clk.mark()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
        t_wall1 = clk.mark()
        if world > 1:
            dist.barrier()
    ms_total = start.elapsed_time(end)
    n_calls, kernel_ms = moe.moe_profile_end()
    if moe.moe_device_status() != 0:
        raise SystemExit("device status not clean after the timed region")
    clocks = clk.summary(t_wall0, t_wall1)
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / args.steps
    value = job_throughput(world, T, args.steps, ms_total)

    # ---------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        x_host = g["x"].cpu().pin_memory()
        out_host = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(g["x"])

        def e2e_step():
            x_dev.copy_(x_host, non_blocking=True)
            layer(x_dev)
            out_host.copy_(out, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e2.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(s2.elapsed_time(e2), world, dev)
        e2e = {"value": job_throughput(world, T, args.steps, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2,
               "ms_per_step": ms_e2e / args.steps}

    # ---------------------------------------------------------- roofline
    peaks, peak_src = load_peaks()
    acc = layer_accounting(cfg, touched, args.weights)
    kname = "gemm_gate_up_swiglu"
    k_ms = kernel_ms.get(kname, 0.0) / max(n_calls, 1)
    # decode and the DeepSeek-V3 shape stream weights (HBM roofline); prefill and
    # the skewed batch are compared with the bf16 tensor peak, as the metric asks
    if args.workload in ("k2_decode", "v3", "tiny"):
        achieved = acc["gate_up_bytes"] / (k_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "kernel": kname,
                "algorithmic_bytes_per_launch": acc["gate_up_bytes"],
                "avg_launch_ms": k_ms, "peak_source": f"{peak_src} hbm_gbs"}
        layer_t = acc["weight_bytes"] / (peak * 1e9)
        layer_roof = {"bound": "hbm", "ideal_ms": layer_t * 1e3, "frac": layer_t / (ms_step / 1e3),
                      "weight_bytes": acc["weight_bytes"], "touched_experts": touched}
    else:
        achieved = acc["gate_up_flops"] / (k_ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        src = f"{peak_src} bf16_tflops_sustained"
        if w8a8:
            # E4M3 x E4M3: the measured bf16 peak times the nominal ratio 4.5 / 2.25
            peak *= 2.0
            src += " x 2 (nominal e4m3 / bf16 ratio)"
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "kernel": kname,
                "algorithmic_flops_per_launch": acc["gate_up_flops"],
                "avg_launch_ms": k_ms, "peak_source": src}
        t_tc = acc["flops"] / (peak * 1e12)
        t_tc_burst = acc["flops"] / (peaks["bf16_tflops"] * (2.0 if w8a8 else 1.0) * 1e12)
        t_hbm = acc["weight_bytes"] / (peaks["hbm_gbs"] * 1e9)
        layer_roof = {"bound": "tensor", "ideal_ms": t_tc * 1e3, "frac": t_tc / (ms_step / 1e3),
                      "hbm_ideal_ms": t_hbm * 1e3, "hbm_frac": t_hbm / (ms_step / 1e3),
                      # the attainable bound: the slower of the weight stream and
                      # the tensor time at the burst peak
                      "attainable_ms": max(t_tc_burst, t_hbm) * 1e3,
                      "attainable_frac": max(t_tc_burst, t_hbm) / (ms_step / 1e3),
                      "flops": acc["flops"], "weight_bytes": acc["weight_bytes"],
                      "touched_experts": touched}
    roof["traffic"] = profiled_traffic(
        args.workload + {"fp8": "_fp8", "w8a8": "_w8a8", "w4a16": "_w4a16"}.get(args.weights, ""),
        kname)

    # ------------------------------------------------ other full-size workloads
    # The default run (the decode headline in bf16) also times the prefill, the
    # skewed and the DeepSeek-V3-shaped batch, one GPU, same process, after the
    # headline's timed region; each has its own steps, clocks and roofline.
    extra = None
    if (world == 1 and not args.no_extra and args.workload == "k2_decode" and not args.set
            and args.weights == "bf16"):
        extra = {"note": "same process, after the headline; weights: the decode run's 384 "
                         "experts (the first 256 for v3), x and bias drawn per workload"}
        for i, name in enumerate(EXTRA_WORKLOADS):
            cfg2, inp = extra_inputs(name, g, dev, seed=1000 + i)
            extra[name] = time_extra_workload(moe, cfg2, inp, dev, args.warmup, peaks, peak_src,
                                              local_rank)
            del inp
        torch.cuda.synchronize(dev)

    # ---------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = OracleSample(cfg, g, args.cpu_sample or default_cpu_sample(cfg, args.weights),
                           args.weights)
        dt = smp.run()
        cpu = {"value": len(smp.tokens) / dt, "unit": UNIT, "cores": smp.threads,
               "kind": "oracle", "sample": smp.describe(), "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if w8a8 else "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload + "".join(f" {x}" for x in args.set),
                       "T": T, "d": d, "E": E, "k": k, "inter": I,
                       "scale": cfg.scale, "bias": cfg.bias, "parallelism": f"replicas{world}",
                       "weights": {"fp8": "fp8_e4m3_block128_pow2",
                                   "w4a16": "int4_group32_sym_bf16_scale",
                                   "w8a8": "w8a8_e4m3_row_pow2"}.get(args.weights, "bf16"),
                       "l2": "inputs larger than L2: every step streams "
                             f"{acc['weight_bytes'] / 1e9:.1f} GB of expert weights"},
            "roofline": roof, "layer_roofline": layer_roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
            "kernel_ms_per_step": {kk: v / max(n_calls, 1) for kk, v in kernel_ms.items()},
        }
        if extra is not None:
            line["workloads"] = extra
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_pdl_ab(moe, args, cfg, step, stream, dev, rounds: int = 4, calls: int = 50):
    """Programmatic dependent launch off and on, alternating in one process: per
    round and setting, a few untimed calls, then `calls` layer calls between two
    CUDA events (no per-kernel events in between: an event recorded between two
    launches orders them and would hide the overlap).  One JSON line with the
    per-round times and their medians."""
    import statistics
    import torch
    res = {False: [], True: []}
    try:
        for _ in range(rounds):
            for pdl in (False, True):
                moe.moe_set_pdl(pdl)
                for _ in range(5):
                    step()
                torch.cuda.synchronize(dev)
                t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                t0.record(stream)
                for _ in range(calls):
                    step()
                t1.record(stream)
                torch.cuda.synchronize(dev)
                res[pdl].append(t0.elapsed_time(t1) / calls)
    finally:
        moe.moe_set_pdl(False)
    if moe.moe_device_status() != 0:
        raise SystemExit("device status not clean after the A/B")
    off, on = statistics.median(res[False]), statistics.median(res[True])
    print(json.dumps({
        "metric": "ms per layer call, programmatic dependent launch off / on",
        "weights": args.weights, "config": {"workload": cfg.name, "T": cfg.T, "E": cfg.E},
        "rounds": rounds, "calls_per_round": calls,
        "off_ms": round(off, 4), "on_ms": round(on, 4),
        "off_rounds": [round(v, 4) for v in res[False]],
        "on_rounds": [round(v, 4) for v in res[True]],
        "gain": round(1.0 - on / off, 4)}))
    return 0


def run_balance(args, cfg):
    """One GPU, one line: the training-side load-balancing pass at the workload's
    shape ("Kimi K2.5 Q&A", Q7.2): unbiased router scores, route, permute, the
    sequence-level balance loss (sequences of S tokens) and the bias update.
    The roofline line is the loss kernels' (token totals, per-block partial
    sums, selection counts, finish): they read the [T, E] fp32 scores twice and
    the [T, k] indices once."""
    import torch
    import sparse_moe_ffn_sigmoid_b200 as moe
    from moe_inputs import make_inputs
    S = args.balance
    T, d, E, k, I = cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter
    if T % S:
        raise SystemExit(f"--balance {S}: T = {T} is not a multiple of S")
    B = T // S
    dev = torch.device("cuda", 0)
    g = make_inputs(cfg, seed=0, device=dev)
    ws = torch.empty(moe.moe_workspace_size(T, d, E, k, I), dtype=torch.uint8, device=dev)
    aux_ws = torch.empty(max(moe.moe_seq_aux_workspace_size(B, S, E), 16), dtype=torch.uint8,
                         device=dev)
    scores = torch.empty((T, E), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    i32 = lambda n: torch.empty((n,), dtype=torch.int32, device=dev)
    counts, offs, rt, sr = i32(E), i32(E + 1), i32(T * k), i32(T * k)
    loss = torch.empty(B, dtype=torch.float32, device=dev)
    bias = g["bias"].clone()
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    aux_ms = []

    def step(timed):
        moe.moe_router_scores(g["x"], g["w_router"], scores, ws)
        moe.moe_route(g["x"], g["w_router"], bias, k, cfg.scale, idx, w, ws)
        moe.moe_permute(idx, E, counts, offs, rt, sr, ws)
        if timed:
            ev[0].record(stream)
        moe.moe_seq_aux_loss(scores, idx, S, 0.001, loss, workspace=aux_ws)
        if timed:
            ev[1].record(stream)
        moe.moe_bias_update(counts, T, k, 1e-3, bias)

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize(dev)
    steps = args.steps or 50
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step(True)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        aux_ms.append(ev[0].elapsed_time(ev[1]))
    total_ms = t0.elapsed_time(t1)
    if moe.moe_device_status() != 0:
        raise SystemExit("device status not clean after the timed region")
    peaks, peak_src = load_peaks()
    aux_bytes = 2 * T * E * 4 + T * k * 4 + T * 4     # scores twice, indices, totals
    a_ms = sum(aux_ms) / len(aux_ms)
    achieved = aux_bytes / (a_ms / 1e3) / 1e9
    line = {"metric": "load-balancing pass tokens/s (router scores, route, permute, "
                      "sequence loss, bias update)",
            "value": T * steps / (total_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
            "steps": steps, "warmup": args.warmup, "ms_per_step": total_ms / steps,
            "higher_is_better": True, "dtype": "fp32", "data": "synthetic",
            "config": {"workload": args.workload, "T": T, "E": E, "k": k, "S": S, "B": B,
                       "note": "each step synchronised to time the loss kernels"},
            "roofline": {"bound": "hbm", "kernel": "seq_aux_loss (4 kernels)",
                         "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "avg_launch_ms": a_ms,
                         "algorithmic_bytes_per_launch": aux_bytes,
                         "peak_source": f"{peak_src} hbm_gbs", "traffic": None},
            "loss": loss.cpu().tolist()}
    print(json.dumps(line), flush=True)
    return 0


REFERENCE_BUDGET_S = 60.0      # target oracle seconds for all warm-up + timed steps


def run_reference(args, cfg, world):
    """The fp64 oracle on the host cores: --warmup + --steps runs of one fixed
    token sample.  The oracle runs one thread per token, so a run takes at
    least one token's time; the sample is a whole number of waves of host
    threads, as many as REFERENCE_BUDGET_S allows (at least one)."""
    import torch
    from moe_inputs import make_inputs
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    g = make_inputs(cfg, seed=0, device=dev)
    runs = args.warmup + args.steps
    if args.cpu_sample:
        n = args.cpu_sample
    else:
        probe = OracleSample(cfg, g, 1, args.weights)   # one token measures the per-token cost
        per_token = probe.run()
        waves = max(1, int(REFERENCE_BUDGET_S / runs / per_token))
        n = max(1, min(cfg.T, waves * host_cores()))
    smp = OracleSample(cfg, g, n, args.weights)
    del g
    per_step = []
    for i in range(runs):
        dt = smp.run()
        if i >= args.warmup:
            per_step.append(dt)
    total = sum(per_step)
    value = len(smp.tokens) * len(per_step) / total
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / len(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": args.workload, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k,
                   "inter": cfg.inter, "scale": cfg.scale, "bias": cfg.bias,
                   "weights": args.weights},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.threads, "kind": "oracle",
                         "sample": smp.describe()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
