"""Benchmark of the shared-experts-fused GLM4-MoE expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_bf16]

One step = one pass of the whole layer (router -> permute -> grouped SwiGLU
GEMMs -> combine) over one batch of the workload, inputs resident in HBM.
Prints one JSON line (rank 0). For N > 1 (torchrun) every rank runs its own
batch with its own copy of the weights (tokens are independent: weak scaling,
no collective on the data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from shared_routed_expert_b200 import MoELayer, _lib, build, synth  # noqa: E402

METRIC = "fused MoE layer tokens/s and TFLOP/s or HBM GB/s vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_PEAKS["hbm_gbs"], "bf16_tflops": FALLBACK_PEAKS["bf16_tflops"],
            "bf16_tflops_sustained": FALLBACK_PEAKS["bf16_tflops"], "source": "fallback"}


# ------------------------------------------------------------------ distributed plumbing

class Dist:
    """One process per GPU (torchrun env). NCCL on GPUs; gloo when no GPU is
    visible (the CPU tests of this host logic). Only the timing barrier and the
    max-over-ranks of the step time are collectives."""

    def __init__(self, gpus: int, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        cuda = torch.cuda.is_available()
        self.backend = backend or ("nccl" if cuda else "gloo")
        self.device = torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {}
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = self.device
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.barrier()
            self.pg.destroy_process_group()


# ------------------------------------------------------------------ clocks

class Clocks:
    """SM clock and clock-event reasons sampled while the timed region runs:
    through NVML every 5 ms (the library nvidia-smi reads), else nvidia-smi
    every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: str):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.thread = None
        self.nvml = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.idx.startswith(("GPU-", "MIG-")):
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.idx)
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.idx))

    def start(self):
        try:
            nv, h = self._nvml_handle()
        except Exception:       # no NVML: fall back to nvidia-smi
            nv = None
        if nv is not None:
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self.nvml = {"sm": [], "reasons": set(), "stop": threading.Event(),
                         "max": nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)}

            def run():
                st = self.nvml
                while not st["stop"].is_set():
                    st["sm"].append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    st["reasons"].update(n for n, b in bits.items() if r & b)
                    st["stop"].wait(0.005)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self) -> dict:
        if self.thread is not None:
            st = self.nvml
            st["stop"].set()
            self.thread.join(timeout=5)
            sm = st["sm"]
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": st["max"],
                    "reasons": sorted(st["reasons"]), "samples": len(sm), "source": "nvml, 5 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sm, smax, reasons = [], None, set()
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower() in ("active", "1"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi, 200 ms"}


# ------------------------------------------------------------------ timing

def emit(line: dict) -> None:
    """Print one JSON line; a figure that was not measured (NaN, e.g. the unfused arm
    under --quick) is written as null so that the line stays strict JSON."""
    def clean(v):
        if isinstance(v, float) and not math.isfinite(v):
            return None
        if isinstance(v, dict):
            return {k: clean(x) for k, x in v.items()}
        if isinstance(v, (list, tuple)):
            return [clean(x) for x in v]
        return v
    print(json.dumps(clean(line), allow_nan=False), flush=True)


def tokens_per_s(n_ranks: int, tokens_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return n_ranks * tokens_per_rank * steps / (max_ms / 1000.0)


def time_steps(fn, steps: int, warmup: int, dist: Dist, stream) -> float:
    """Device time of `steps` back-to-back calls (ms), max over ranks."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    return dist.max(e0.elapsed_time(e1))


KERNELS = ["route_logits", "route_split", "route_approx", "route_candidates", "route_verify", "route_topk",
           "permute_small", "permute_hist", "permute_scan", "permute_scatter", "permute_fused",
           "quant_x", "quant_h", "gather", "gemm1_tc", "gemm2_tc", "gemm1_simt", "gemm2_simt", "combine"]

RV_MAXC = 32            # candidate slots per token of the verified tensor-core routing


def route_tc_path(cfg) -> bool:
    """Whether moe_forward routes through approximate tensor-core logits verified
    exactly (renormalised top-K over bf16 activations, batches over 256 tokens,
    32..256 routed experts, K <= 16, H <= 8192), as the library decides."""
    return (cfg.act_dtype == "bf16" and cfg.renormalize and cfg.T > 256 and 32 <= cfg.n_routed <= 256
            and cfg.top_k <= 16 and cfg.H % 256 == 0 and cfg.H <= 8192)


def route_tc_dims(cfg):
    """(NP, KS): expert rows padded to 32 and the number of H slices of the
    approximate logits."""
    nkb, nseg = cfg.H // 64, cfg.H // 256
    ks = 4 if (nseg >= 4 and nkb % 4 == 0) else (2 if (nseg >= 2 and nkb % 2 == 0) else 1)
    return (cfg.n_routed + 31) // 32 * 32, ks


def kernel_table(steps: int) -> dict:
    tab = {}
    total = 0.0
    for k in KERNELS:
        n, ms = _lib.moe_profile_read(k)
        if n:
            tab[k] = {"launches": n, "total_ms": ms, "ms_per_launch": ms / n}
            total += ms
    for k in tab:
        tab[k]["share"] = tab[k]["total_ms"] / total if total > 0 else None
    return tab


def token_major_gather(cfg) -> bool:
    """The layer gathers its rows token by token (bf16 tokens on the tensor-core
    path, at least 1024 of them, H <= 5120), quantising them there for E4M3 weights."""
    return (cfg.act_dtype == "bf16" and cfg.w_dtype != "f32" and cfg.T >= 1024 and cfg.H % 8 == 0
            and cfg.H <= 5120)


def algorithmic(cfg, kernel: str, counts: np.ndarray | None, fused: bool = True):
    """(flops, bytes) one launch of `kernel` must do for this workload: flops of
    the dense contraction it performs (None if it is not one), and the bytes it
    must move at least once (touched experts' weights, its own inputs/outputs)."""
    R, T, H, I, Er = cfg.rows, cfg.T, cfg.H, cfg.I, cfg.n_routed
    E = cfg.n_experts
    wb = 1 if cfg.w_dtype == "e4m3" else (4 if cfg.w_dtype == "f32" else 2)
    ab = 4 if cfg.act_dtype == "f32" else 2
    xb = 1 if wb == 1 else ab                      # bytes per GEMM input activation
    touched = int((counts > 0).sum()) if counts is not None else cfg.n_experts
    n_chunks = -(-R // 512)                        # 512-slot chunks of the permutation
    if kernel.startswith("gemm1"):
        return 2.0 * R * 2 * I * H, touched * 2 * I * H * wb + R * H * xb + R * I * ab
    if kernel.startswith("gemm2"):
        # reads h, writes the expert rows y as scaled fp16 plus one exponent byte per 32 columns
        return 2.0 * R * I * H, touched * H * I * wb + R * I * xb + R * H * 2 + R * (H // 32)
    if kernel == "route_logits":
        return None, T * H * ab + Er * H * 4 + (H // 256) * T * Er * 4
    NP, KS = route_tc_dims(cfg)
    if kernel == "route_split":
        # fp32 router weights in, their bf16 high and low parts out
        return None, Er * H * 4 + 2 * NP * H * 2
    if kernel == "route_approx":
        # two bf16 GEMMs (x times the high and the low parts); x and the split
        # weights in, KS fp32 slices of the approximate logits out
        return 2.0 * T * 2 * NP * H, T * H * ab + 2 * NP * H * 2 + KS * T * Er * 4
    if kernel == "route_candidates":
        # the slices and x (for its norm) in, the candidate lists out (and each
        # pair's entry in its expert's bucket, at most RV_MAXC per token)
        return None, KS * T * Er * 4 + T * H * ab + T * (1 + RV_MAXC) * 4
    if kernel == "route_verify":
        # x and the router weights once, the bucketed pairs (at most RV_MAXC per
        # token) in; the candidates' segment partials out
        return None, T * H * ab + Er * H * 4 + T * (1 + RV_MAXC) * 4 + (H // 256) * T * RV_MAXC * 4
    if kernel == "route_topk":
        # the segment partials (all experts', or the candidates') in; ids and weights out
        per_token = RV_MAXC if route_tc_path(cfg) else Er
        return None, (H // 256) * T * per_token * 4 + R * 8
    if kernel == "combine":
        return None, R * H * 2 + R * (H // 32) + T * H * ab + R * 4 * 2
    if kernel == "gather":
        # the fused layer's shared rows are read from x by GEMM1 and not copied:
        # x read once, the routed rows written (plus per-row scales for E4M3)
        copied = R - T if (fused and cfg.shared) else R
        if wb == 1 and token_major_gather(cfg):
            # bf16 x read once, quantised: the token codes and the routed rows' codes written
            return None, T * H * ab + (T + copied) * (H + 4)
        return None, T * H * xb + copied * H * xb + (copied * 4 + T * 4 if wb == 1 else 0)
    if kernel == "quant_x":
        # x per token (T rows of H): bf16 in, E4M3 codes and one scale per row out
        return None, T * H * 3 + T * 4
    if kernel == "quant_h":
        # h per permuted row (R rows of I)
        return None, R * I * 3 + R * 4
    if kernel == "permute_small":
        return None, R * 4 + 2 * R * 4 + (2 * E + 1) * 4
    if kernel == "permute_hist":
        return None, R * 4 + n_chunks * E * 4
    if kernel == "permute_scan":
        return None, 2 * n_chunks * E * 4 + 3 * (E + 1) * 4
    if kernel == "permute_scatter":
        return None, R * 4 + n_chunks * E * 4 + (E + 1) * 4 + 2 * R * 4
    if kernel == "permute_fused":
        # ids in, perm and inv out, the chunk counts written once and read back once
        return None, R * 4 + 2 * R * 4 + 2 * n_chunks * E * 4 + 3 * (E + 1) * 4
    return None, None


# DRAM bytes (read + write) / algorithmic bytes of one launch, from one ncu
# capture of the same kernel variant on a 32-routed-expert case of the workload
# the variant serves (1024 tokens of prefill_bf16 or prefill_fp8, whose
# per-expert row counts match the full ones; the 64-token decode batch). Traffic
# is dominated by the touched experts' weights, so it scales with the launch.
# Keyed by (kernel, weight dtype, tensor-core work unit).
PROFILED_TRAFFIC_RATIO = {("gemm1_tc", "bf16", "swap"): 1.007, ("gemm2_tc", "bf16", "pair256x512"): 0.967,
                          ("gemm1_tc", "bf16", 128): 1.009, ("gemm2_tc", "bf16", 128): 0.998,
                          ("gemm1_tc", "e4m3", 128): 1.002, ("gemm2_tc", "e4m3", 128): 0.911}


def unit_rows(cfg, ffn: str, kernel: str = "gemm1_tc"):
    """Tensor-core work unit `kernel` uses in the run: 128, 256 (one CTA),
    "pair256" (256 x 256 tiles over a CTA pair), "pair256x512" (256 x 512 pair
    tiles) or "swap" (CTA pairs, 256 weight rows x up to 256 tokens)."""
    if ffn == "tcgen05_m128":
        return 128
    if ffn == "tcgen05_m256":
        return 256
    if ffn == "tcgen05_pair":
        return "pair256"
    if ffn == "tcgen05_wide":
        return "pair256x512"
    if ffn == "tcgen05_swap":
        return "swap"
    if cfg.w_dtype == "bf16" and cfg.rows >= 192 * cfg.n_experts:
        return "swap" if (kernel == "gemm1_tc" and cfg.I % 256 == 0) else "pair256x512"
    return 128


def roofline_of(cfg, kernel: str, ms_per_launch: float, counts, pk, ffn: str = "auto") -> dict:
    flops, nbytes = algorithmic(cfg, kernel, counts)
    ratio = PROFILED_TRAFFIC_RATIO.get((kernel, cfg.w_dtype, unit_rows(cfg, ffn, kernel)))
    traffic = int(ratio * nbytes) if (ratio and nbytes) else None
    t = ms_per_launch / 1000.0
    tpk = pk["bf16_tflops"] * (2.0 if cfg.w_dtype == "e4m3" else 1.0)
    src = f"{pk['source']} bf16 {pk.get('tensor_label', 'burst')}" + \
        (" x2 (E4M3/bf16 nominal ratio)" if cfg.w_dtype == "e4m3" else "")
    if kernel == "route_logits":
        # fp32 CUDA-core FMAs in a fixed order (2 flop each)
        fl = 2.0 * cfg.T * cfg.n_routed * cfg.H
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        return {"kernel": kernel, "bound": "alu", "achieved": fl / t / 1e12, "peak": peak,
                "unit": "TFLOP/s", "frac": fl / t / 1e12 / peak, "traffic": None,
                "peak_source": "148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz"}
    t_tensor = flops / (tpk * 1e12) if flops else 0.0
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9) if nbytes else 0.0
    if flops and t_tensor >= t_hbm:
        ach = flops / t / 1e12
        return {"kernel": kernel, "bound": "tensor", "achieved": ach, "peak": tpk, "unit": "TFLOP/s",
                "frac": ach / tpk, "traffic": traffic, "peak_source": src,
                "hbm_frac": nbytes / t / 1e9 / pk["hbm_gbs"]}
    ach = (nbytes or 0) / t / 1e9
    out = {"kernel": kernel, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
           "frac": ach / pk["hbm_gbs"], "traffic": traffic, "peak_source": pk["source"],
           "algorithmic_bytes": nbytes}
    if flops:
        out["tensor_frac"] = flops / t / 1e12 / tpk
    return out


# ------------------------------------------------------------------ CPU oracle baseline

def cpu_baseline(cfg, host_inputs: dict, seconds: float = 12.0):
    import oracle
    Ly = oracle.Layer(cfg, host_inputs)
    cores = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(0)
    n = max(1, cores)
    tok = rng.choice(cfg.T, size=min(n, cfg.T), replace=False).astype(np.int32)
    t0 = time.perf_counter()
    r = Ly.forward(tokens=tok, n_threads=cores)
    dt = time.perf_counter() - t0
    done, used = len(tok), r["threads"]
    # scale the sample up to roughly `seconds` of CPU work
    more = int(min(cfg.T - len(tok), max(0, len(tok) * (seconds / max(dt, 1e-3) - 1.0))))
    if more > 0:
        tok2 = rng.choice(np.setdiff1d(np.arange(cfg.T), tok), size=more, replace=False).astype(np.int32)
        t1 = time.perf_counter()
        r = Ly.forward(tokens=tok2, n_threads=cores)
        dt += time.perf_counter() - t1
        done += more
        used = max(used, r["threads"])
    out = {"value": done / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
           "sample": f"{done} tokens of {cfg.name} (router + all {cfg.slots} slots each, fp64 C oracle), {dt:.1f} s"}
    if cfg.T <= 64:
        # small batches are also timed on one core: up to 8 tokens, once
        tok1 = rng.choice(cfg.T, size=min(8, cfg.T), replace=False).astype(np.int32)
        t1 = time.perf_counter()
        Ly.forward(tokens=tok1, n_threads=1)
        dt1 = time.perf_counter() - t1
        out["single_thread"] = {"value": len(tok1) / dt1, "unit": "tokens/s", "cores": 1,
                                "sample": f"{len(tok1)} tokens of {cfg.name}, {dt1:.2f} s"}
    return out


def run_reference(args, dist: Dist):
    """The reference arm: the CPU oracle as it stands, bounded sample per step."""
    if dist.rank != 0:
        return
    import oracle
    cfg = synth.CONFIGS[args.workload]
    host = synth.to_host(synth.make_inputs(cfg, dist.device))
    Ly = oracle.Layer(cfg, host)
    cores = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(1)
    per_step = max(1, cores)

    def step():
        tok = rng.choice(cfg.T, size=per_step, replace=False).astype(np.int32)
        return Ly.forward(tokens=tok, n_threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    used = 1
    for _ in range(args.steps):
        used = max(used, step()["threads"])
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(cfg), "sample_tokens_per_step": per_step},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "sample": f"{per_step} random tokens of {cfg.name} per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    emit(line)


def describe(cfg) -> str:
    return (f"{cfg.name}: T={cfg.T} H={cfg.H} I={cfg.I} {cfg.n_routed} routed + shared as expert "
            f"{cfg.shared_id}, top-{cfg.top_k} + shared slot, {cfg.w_dtype} weights, {cfg.act_dtype} "
            f"activations, seed {cfg.seed}")


# ------------------------------------------------------------------ main

def bench_tp(args, dist):
    """Tensor-parallel layer: each of the N ranks holds 1/N of every expert's
    intermediate dimension and the ranks sum their fp32 shares with one NCCL
    all-reduce of [T, H] (strong scaling: the layer is fixed, N GPUs share it)."""
    from shared_routed_expert_b200 import tp
    N = dist.world
    cfg = synth.CONFIGS[args.workload]
    if cfg.I % N or (cfg.I // N) % 64:
        raise SystemExit(f"I = {cfg.I} does not split into {N} slices of a multiple of 64")
    full = synth.make_inputs(cfg, "cpu")
    shard = synth.to_device(tp.shard_weights(full, cfg.I, dist.rank, N), dist.device)
    x = full["x"].to(dist.device)
    del full
    layer = tp.TPMoELayer(cfg, shard, N)          # the default process group: the N ranks
    stream = torch.cuda.current_stream()
    ms = time_steps(lambda: layer.forward(x), args.steps, args.warmup, dist, stream)
    line = {"metric": "tensor-parallel MoE layer tokens/s", "value": cfg.T * args.steps / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": N, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": cfg.w_dtype, "data": "synthetic",
            "config": {"workload": describe(cfg), "parallelism": f"tp{N} (intermediate slices of {cfg.I // N}, "
                                                               "one fp32 all-reduce of [T, H] per layer)"}}
    if dist.rank == 0:
        emit(line)


def bench_qk_norm_rope(args, dist):
    line = measure_qk_norm_rope(synth.ATTN_CONFIGS[args.attn_workload], args, dist)
    if dist.rank == 0:
        emit(line)


def measure_qk_norm_rope(cfg, args, dist) -> dict:
    """The fused QK-norm + partial RoPE kernel on its own: tokens/s from the
    kernel's CUDA events (L2 flushed between launches by an untimed 256 MB
    read, which leaves no dirty lines to write back during the kernel), rated
    against the measured HBM copy peak; e2e uploads qkv and downloads it every
    step."""
    inp = synth.make_attn_inputs(cfg, dist.device)
    stream = torch.cuda.current_stream()
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dist.device)

    def launch(qkv):
        _lib.moe_qk_norm_rope(cfg, qkv, inp["pos"], inp["q_w"], inp["k_w"], inp["cos_sin"])

    def step():
        flush.amax()
        launch(inp["qkv"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    clocks = Clocks(vis.split(",")[dist.local] if vis else str(dist.local))
    n0 = _lib.moe_launch_count()
    _lib.moe_profile_reset()
    _lib.moe_profile_enable(True)
    clocks.start()
    time_steps(step, args.steps, 0, dist, stream)
    clk = clocks.stop()
    _lib.moe_profile_enable(False)
    launches = _lib.moe_launch_count() - n0
    n, tot = _lib.moe_profile_read("qk_norm_rope")
    ms_launch = dist.max(tot / max(n, 1))
    # end to end: pinned host qkv up, kernel, qkv down, every step
    host_in = inp["qkv"].cpu().pin_memory()
    host_out = torch.empty_like(host_in).pin_memory()
    dev = torch.empty_like(inp["qkv"])

    def e2e_step():
        dev.copy_(host_in, non_blocking=True)
        launch(dev)
        host_out.copy_(dev, non_blocking=True)
    ms_e2e = time_steps(e2e_step, args.steps, args.warmup, dist, stream)
    pk = peaks()
    nbytes = cfg.moved_bytes()
    ach = nbytes / (ms_launch / 1e3) / 1e9
    N = dist.world
    line = {
        "metric": "fused QK-norm + partial RoPE tokens/s vs B200 HBM roofline", "op": "qk_norm_rope",
        "value": N * cfg.T / (ms_launch / 1e3), "unit": "tokens/s", "n_gpus": N, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_launch, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: T={cfg.T} q heads {cfg.n_q}, kv heads {cfg.n_kv}, head_dim {cfg.d}, "
                               f"rotated {cfg.rot}, positions {'0..T-1' if cfg.sequential else 'random'}",
                   "l2": "flushed between launches (256 MB read, not timed)"},
        "e2e": {"value": N * cfg.T * args.steps / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": host_in.numel() * 2, "d2h_bytes_per_step": host_out.numel() * 2},
        "gpu_launches": int(launches),
        "roofline": {"kernel": "qk_norm_rope", "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": ach / pk["hbm_gbs"], "traffic": None, "peak_source": pk["source"],
                     "algorithmic_bytes": nbytes},
        "clocks": clk,
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_bf16", choices=list(synth.CONFIGS))
    ap.add_argument("--ffn", default="auto",
                    choices=["auto", "simt", "tcgen05", "tcgen05_m128", "tcgen05_m256", "tcgen05_pair",
                             "tcgen05_wide", "tcgen05_swap"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only --workload (by default the other workloads follow in a 'workloads' object)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--quick", action="store_true",
                    help="only the fused device-timed region (for ncu launch lists and captures)")
    ap.add_argument("--tokens", type=int, default=None, help="override T (smaller profiling case)")
    ap.add_argument("--routed", type=int, default=None, help="override the routed expert count")
    ap.add_argument("--inter", type=int, default=None, help="override I (smaller profiling case)")
    ap.add_argument("--op", default="moe", choices=["moe", "qk_norm_rope"],
                    help="moe: the expert layer (default); qk_norm_rope: the attention pre-processing kernel")
    ap.add_argument("--attn-workload", default="qknorm_prefill", choices=list(synth.ATTN_CONFIGS))
    ap.add_argument("--tp", action="store_true",
                    help="tensor parallelism over the launched ranks instead of replicas")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    dist = Dist(args.gpus)
    torch.cuda.set_device(dist.device)
    if args.impl == "reference":
        run_reference(args, dist)
        dist.close()
        return

    build.build()
    if args.op == "qk_norm_rope":
        bench_qk_norm_rope(args, dist)
        dist.close()
        return
    if args.tp:
        bench_tp(args, dist)
        dist.close()
        return
    cfg = synth.CONFIGS[args.workload]
    if args.tokens is not None or args.routed is not None or args.inter is not None:
        cfg = synth.variant(cfg, T=args.tokens or cfg.T, n_routed=args.routed or cfg.n_routed,
                            I=args.inter or cfg.I,
                            name=f"{cfg.name}[T={args.tokens or cfg.T},E_r={args.routed or cfg.n_routed},"
                                 f"I={args.inter or cfg.I}]")
    impl = {"auto": _lib.MOE_FFN_AUTO, "simt": _lib.MOE_FFN_SIMT, "tcgen05": _lib.MOE_FFN_TCGEN05,
            "tcgen05_m128": _lib.MOE_FFN_TCGEN05_M128, "tcgen05_m256": _lib.MOE_FFN_TCGEN05_M256,
            "tcgen05_pair": _lib.MOE_FFN_TCGEN05_PAIR, "tcgen05_wide": _lib.MOE_FFN_TCGEN05_WIDE,
            "tcgen05_swap": _lib.MOE_FFN_TCGEN05_SWAP}[args.ffn]
    N = dist.world
    base = dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline
    m = measure(cfg, args, dist, impl, quick=args.quick, want_host=base and not args.quick)
    line = {
        "metric": METRIC, "value": m["value"], "unit": "tokens/s", "n_gpus": N, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.w_dtype == "bf16" else cfg.w_dtype,
        "data": "synthetic",
        "config": {"workload": describe(cfg), "global_batch_tokens": N * cfg.T,
                   "parallelism": f"replicas x{N} (tokens sharded, weights replicated)",
                   "l2": "inputs larger than L2: every step streams the touched experts' weights "
                         f"({m['alg_bytes'] / 1e9:.2f} GB) through the 126 MB L2",
                   "ffn_impl": args.ffn},
        "tflops": m["tflops"], "tensor_frac": m["tensor_frac"], "hbm_gbs": m["hbm_gbs"], "hbm_frac": m["hbm_frac"],
        "fused_speedup": m["unfused"]["fused_speedup"],
        "unfused": m["unfused"],
        "combine_fold": m["combine_fold"],
        "e2e": m["e2e"],
        "gpu_launches": m["gpu_launches"],
        "roofline": m["roofline"],
        "kernels": m["kernels"],
        "clocks": m["clocks"],
        "peaks": m["peaks"],
    }
    if base and not args.quick:
        line["cpu_baseline"] = cpu_baseline(cfg, m["host"], args.cpu_seconds)
    m.pop("host", None)
    # the other workloads of the layer, measured the same way in the same run
    extra = [] if (args.quick or args.no_workloads) else [w for w in WORKLOADS if w != cfg.name]
    if extra:
        line["workloads"] = {}
        for name in extra:
            wcfg = synth.CONFIGS[name]
            wm = measure(wcfg, args, dist, impl, quick=False, want_host=base and wcfg.T <= 64)
            entry = {"workload": describe(wcfg), "value": wm["value"], "unit": "tokens/s",
                     "ms_per_step": wm["ms_per_step"], "steps": args.steps,
                     "tflops": wm["tflops"], "tensor_frac": wm["tensor_frac"], "hbm_gbs": wm["hbm_gbs"],
                     "hbm_frac": wm["hbm_frac"], "roofline": wm["roofline"],
                     "fused_speedup": wm["unfused"]["fused_speedup"], "unfused": wm["unfused"],
                     "combine_fold": wm["combine_fold"],
                     "e2e": wm["e2e"], "gpu_launches": wm["gpu_launches"], "clocks": wm["clocks"],
                     "kernels": {k: {kk: v[kk] for kk in ("launches", "ms_per_launch", "share", "roofline")}
                                 for k, v in wm["kernels"].items()}}
            if base and wcfg.T <= 64:
                entry["cpu_baseline"] = cpu_baseline(wcfg, wm["host"], args.cpu_seconds / 2)
            wm.pop("host", None)
            line["workloads"][name] = entry
            del wm
            torch.cuda.empty_cache()
        # the attention-side step the pages fuse (QK-norm + partial RoPE), prefill and decode
        for name in ("qknorm_prefill", "qknorm_decode"):
            q = measure_qk_norm_rope(synth.ATTN_CONFIGS[name], args, dist)
            line["workloads"][name] = {k: q[k] for k in ("metric", "value", "unit", "ms_per_step", "steps", "config",
                                                          "e2e", "gpu_launches", "roofline", "clocks")}
            torch.cuda.empty_cache()
    if dist.rank == 0:
        emit(line)
    dist.close()


WORKLOADS = ["prefill_bf16", "decode_bf16", "prefill_fp8", "skewed_fp8"]


def measure(cfg, args, dist: Dist, impl: int, quick: bool = False, want_host: bool = False) -> dict:
    """Everything one workload reports: the fused layer device-timed over
    args.steps back-to-back steps (inputs resident in HBM, per-kernel events on
    the launching stream), the unfused layer in interleaved blocks, and the end
    to end path through host buffers."""
    d = synth.make_inputs(cfg, dist.device)
    stream = torch.cuda.current_stream(dist.device)
    fused = MoELayer(cfg, d, fuse_shared=True, impl=impl)
    out = torch.empty_like(d["x"])

    # expert counts of this batch (for touched-expert bytes)
    s = _lib.make_shape(cfg)
    ids = torch.empty(cfg.T, cfg.slots, dtype=torch.int32, device=dist.device)
    wts = torch.empty(cfg.T, cfg.slots, dtype=torch.float32, device=dist.device)
    _lib.moe_route_topk(s, d["x"], d["router_w"], d["router_bias"], ids, wts, None, fused.ws)
    counts = np.bincount(ids.cpu().numpy().ravel(), minlength=cfg.n_experts)

    def step():
        fused.forward(d["x"], out)

    # timed region: device-resident inputs, the layer's kernels back to back with
    # nothing between them (a kernel may start while its predecessor finishes)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    clocks = Clocks(vis.split(",")[dist.local] if vis else str(dist.local))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    n0 = _lib.moe_launch_count()
    clocks.start()
    ms = time_steps(step, args.steps, 0, dist, stream)
    clk = clocks.stop()
    launches = _lib.moe_launch_count() - n0
    # per-kernel durations: a second pass of as many steps with CUDA events
    # around every launch on the launching stream (these serialise the kernels)
    _lib.moe_profile_reset()
    _lib.moe_profile_enable(True)
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    _lib.moe_profile_reset()
    time_steps(step, args.steps, 0, dist, stream)
    _lib.moe_profile_enable(False)
    tab = kernel_table(args.steps)
    st = fused.status()
    if st != _lib.MOE_OK:
        raise SystemExit(f"{cfg.name}: layer reported {_lib.status_string(st)}")

    if quick:
        ms_unf = ms_e2e = ms_fused_il = ms_sep = float("nan")
        unf_steps = args.steps
        n_blocks, per = 0, 0
        tab_unf = {}
        x_host = out_host = d["x"]
    else:
        # unfused GPU baseline (shared expert as its own dense pass), same process,
        # timed in blocks interleaved with blocks of the fused layer so that both
        # see the same clocks (the power cap moves them by several percent over
        # a run); per-kernel events on during the unfused blocks only
        unfused = MoELayer(cfg, d, fuse_shared=False, impl=impl)
        # the fused layer with its weighted aggregation inside the down-projection
        # (opt-in: measured slower than the separate pass)
        separate = MoELayer(cfg, d, fuse_shared=True, impl=impl | _lib.MOE_FFN_COMBINE_FOLD)
        for _ in range(args.warmup):
            unfused.forward(d["x"], out)
            separate.forward(d["x"], out)
        torch.cuda.synchronize()
        _lib.moe_profile_reset()
        n_blocks = max(1, min(10, args.steps))
        per = max(1, args.steps // n_blocks)
        ms_unf = ms_fused_il = ms_sep = 0.0
        for _ in range(n_blocks):
            ms_fused_il += time_steps(step, per, 0, dist, stream)
            ms_unf += time_steps(lambda: unfused.forward(d["x"], out), per, 0, dist, stream)
            ms_sep += time_steps(lambda: separate.forward(d["x"], out), per, 0, dist, stream)
        unf_steps = n_blocks * per
        # the unfused layer's per-kernel durations, in a pass of its own with events
        _lib.moe_profile_reset()
        _lib.moe_profile_enable(True)
        time_steps(lambda: unfused.forward(d["x"], out), unf_steps, 0, dist, stream)
        _lib.moe_profile_enable(False)
        tab_unf = kernel_table(unf_steps)
        for lay, what in ((unfused, "unfused"), (separate, "folded combine")):
            st = lay.status()
            if st != _lib.MOE_OK:
                raise SystemExit(f"{cfg.name} {what}: layer reported {_lib.status_string(st)}")
        del unfused, separate

        # end to end through the public API with pinned host buffers: every step
        # uploads its x and downloads its out; the pipelined submission overlaps
        # one step's copies with its neighbours' compute
        x_host = d["x"].cpu().pin_memory()
        out_hosts = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
        for i in range(args.warmup):
            fused.submit_host(x_host, out_hosts[i % 2])
        fused.sync_host()
        dist.barrier()
        h2d, comp, d2h = fused.host_streams()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(h2d)
        for i in range(args.steps):
            fused.submit_host(x_host, out_hosts[i % 2])
        e1.record(d2h)           # after the last download, which depends on every earlier step
        fused.sync_host()
        dist.barrier()
        ms_e2e = dist.max(e0.elapsed_time(e1))
        out_host = out_hosts[0]
    N = dist.world
    ms_step = ms / args.steps
    pk = peaks()
    flops = cfg.gemm_flops() + cfg.router_flops()
    wb = 1 if cfg.w_dtype == "e4m3" else 2
    alg_bytes = int((counts > 0).sum()) * 3 * cfg.H * cfg.I * wb + 2 * cfg.T * cfg.H * 2 + \
        cfg.n_routed * cfg.H * 4
    # kernels timed inside a long loop run under the 1 kW power cap: their tensor
    # peak is the measured sustained cuBLAS figure, the burst one otherwise
    if ms >= 250.0:
        pk = dict(pk, bf16_tflops=pk["bf16_tflops_sustained"], tensor_label="sustained")
    tensor_peak = pk["bf16_tflops"] * (2.0 if cfg.w_dtype == "e4m3" else 1.0)

    roof = None
    if tab:
        top = max(tab, key=lambda k: tab[k]["total_ms"])
        roof = roofline_of(cfg, top, tab[top]["ms_per_launch"], counts, pk, args.ffn)
        for k in tab:
            tab[k]["roofline"] = roofline_of(cfg, k, tab[k]["ms_per_launch"], counts, pk, args.ffn)
    host = synth.to_host(d) if want_host else None
    res = {
        "value": tokens_per_s(N, cfg.T, args.steps, ms), "ms_per_step": ms_step, "alg_bytes": alg_bytes,
        "tflops": flops / (ms_step / 1000.0) / 1e12,
        "tensor_frac": flops / (ms_step / 1000.0) / 1e12 / tensor_peak,
        "hbm_gbs": alg_bytes / (ms_step / 1000.0) / 1e9,
        "hbm_frac": alg_bytes / (ms_step / 1000.0) / 1e9 / pk["hbm_gbs"],
        "unfused": {"value": N * cfg.T * unf_steps / (ms_unf / 1000.0), "ms_per_step": ms_unf / unf_steps,
                    "fused_ms_per_step_interleaved": ms_fused_il / unf_steps,
                    "fused_speedup": ms_unf / ms_fused_il,
                    "timing": f"{n_blocks} blocks of {per} steps, fused and unfused alternating",
                    "kernels": {k: {"launches": v["launches"], "ms_per_step": v["total_ms"] / unf_steps}
                                for k, v in tab_unf.items()}},
        "combine_fold": {"ms_per_step": ms_sep / unf_steps,
                         "fold_speedup": ms_fused_il / ms_sep,
                         "timing": "the fused layer with its aggregation inside the down-projection "
                                   "(MOE_FFN_COMBINE_FOLD), in the same alternating blocks; fold_speedup "
                                   "= default (separate pass) time / folded time"},
        "e2e": {"value": N * cfg.T * args.steps / (ms_e2e / 1000.0), "unit": "tokens/s",
                "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
                "d2h_bytes_per_step": out_host.numel() * out_host.element_size()},
        "gpu_launches": int(launches), "roofline": roof, "kernels": tab, "clocks": clk, "peaks": pk,
        "host": host,
    }
    del fused, d
    return res


if __name__ == "__main__":
    main()
