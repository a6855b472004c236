#!/usr/bin/env python
"""Throughput of the FLARE++ mixer forward on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one full forward call (synthesis, gate, encode, decode: every
launch of the hot path) over one batch of the workload's synthetic inputs,
already resident in HBM.  The default workload is the 1M-token scaling case
(B=1, H=8, N=1048576, M=512, D=64, bf16); its inputs (1 GiB per [B,H,N,D]
tensor) are larger than the 126 MB L2, so steps run back to back.  Smaller
workloads get an L2 flush (a 512 MiB write) between steps and the step times
are summed.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
problem of the same size (weak scaling, no collective on the data path); the
timed region is bracketed by a barrier and a device synchronise, the elapsed
device time is the maximum over ranks, and ``value`` counts the tokens of all
ranks.

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FLARE++ mixer fwd Mtokens/s on 1 B200 + % of roofline (HBM GB/s or TFLOP/s)"
UNIT = "Mtokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES_GATED = ["split_partial(synthesis)", "merge(q)", "split_partial(encode)", "merge(z)", "decode"]
STAGES_FLARE = ["split_partial(encode)", "merge(z)", "decode"]


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="scale1m_bf16")
    p.add_argument("--tokens", type=int, default=0,
                   help="override N of the workload (a smaller case of the same kernels, e.g. for ncu)")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--path", choices=["auto", "simt", "tcgen05"], default="auto")
    p.add_argument("--flare", action="store_true", help="closed gate: the two-call FLARE form (flare_fwd)")
    p.add_argument("--norm", action="store_true",
                   help="RMS-normalise q0 and k0 rows inside the synthesis pass (norm_synthesis)")
    p.add_argument("--cp", action="store_true",
                   help="token-sharded form: one global problem, each rank holds N/world tokens (strong scaling)")
    p.add_argument("--layout", choices=["bhnd", "bnhd"], default="bhnd",
                   help="memory layout of k0, k, v, y: [B,H,N,D] or [B,N,H,D] (read in place)")
    p.add_argument("--backward", action="store_true",
                   help="time the backward (flarepp_mixer_bwd: gradients of every input for a random dy)")
    p.add_argument("--saved-state", action="store_true",
                   help="with --backward: time the backward from a training forward's saved state "
                        "(flarepp_mixer_bwd_ctx; the forward runs once, untimed)")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the per-configuration record (every BASELINE workload timed and checked "
                        "against the oracle on rank 0)")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return p.parse_args(argv)


# --------------------------------------------------------------------------- ranks

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own problem (independent batches: weak scaling)."""
    return base_seed + 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity on one rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_mtokens(tokens_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: tokens processed by all ranks over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / (max_ms * 1e-3) / 1e6


# --------------------------------------------------------------------------- peaks, clocks, traffic

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {"split_partial": ["common.cuh", "kernels_tc.cuh"]}


def code_only(src: str) -> str:
    """C++/CUDA source without its comments, whitespace runs collapsed to one
    space; string and character literals are kept as written."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_digest(kernel: str = "split_partial") -> str:
    """Digest of the code of the source files that define a kernel, comments
    left out (so a recorded ncu traffic figure is used only for the code it was
    measured on, and an edited comment does not retire it)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_latent_attention_mixer_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update((name + "\n" + code_only(f.read())).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, only if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_digest") != source_digest(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock, max clock, utilisation and clock-event reasons through
    NVML every `period` seconds while running (read-only queries)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period: float = 0.005):
        self.period = period
        self.samples = []
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            self.nvml = pynvml
            pynvml.nvmlInit()
            self.handle = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = repr(e)
            self.handle = None
            self.max_mhz = None

    def _handle(self, device_index):
        import torch
        pynvml = self.nvml
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        pynvml = self.nvml
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
                util = pynvml.nvmlDeviceGetUtilizationRates(self.handle).gpu
                try:
                    reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                except AttributeError:
                    reasons = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                self.samples.append((sm, util, reasons))
            except Exception as e:  # pragma: no cover
                self.error = repr(e)
            self._stop.wait(self.period)

    def __enter__(self):
        if self.handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.error}
        loaded = [s for s in self.samples if s[1] >= 50] or self.samples
        reasons = set()
        for _, _, r in loaded:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "samples_under_load": len(loaded)}


# --------------------------------------------------------------------------- CPU oracle sample

def oracle_sample(x_cpu_head, w, n_tokens: int):
    """Times the oracle on one (b, h) slice restricted to the first n_tokens
    tokens: synthesis and encode over those tokens, decode of every one."""
    import numpy as np
    import oracle
    sl = slice(0, n_tokens)
    q0, qf, g, k0, k, v = x_cpu_head
    toks = np.arange(n_tokens, dtype=np.int64)
    args = (q0, qf, g, k0[sl], k[sl], v[sl], toks)
    t0 = time.perf_counter()
    oracle.flarepp_head(*args)
    return time.perf_counter() - t0


def head_slice_cpu(x, w):
    return (x["q0"][0].cpu(), x["q_fixed"][0].cpu(), float(x["gate"][0]), x["k0"][0, 0].cpu(),
            x["k"][0, 0].cpu(), x["v"][0, 0].cpu())


def cpu_baseline(x, w, target_s: float):
    """Bounded sample of the workload on the host cores; returns the entry and
    the per-step sample size.  Tokens/s covers all H heads of the workload:
    the sample runs one head, so its per-token time is multiplied by H."""
    import oracle
    head = head_slice_cpu(x, w)
    n_cal = min(w.N, 1024)
    t_cal = oracle_sample(head, w, n_cal)
    per_tok = max(t_cal / n_cal, 1e-9)
    n = int(min(w.N, max(n_cal, target_s / per_tok)))
    t = oracle_sample(head, w, n)
    value = n / (t * w.H) / 1e6 if t > 0 else None
    return {
        "value": value,
        "unit": UNIT,
        "cores": oracle.num_threads(),
        "kind": "oracle",
        "sample": (f"{w.name}: batch 0, head 0 of {w.H}, first {n} of {w.N} tokens, all M={w.M} latents, "
                   f"D={w.D}, fp64; synthesis and encode over the sample, every sample token decoded; "
                   f"tokens/s = sample tokens / (time x {w.H} heads)"),
        "seconds": t,
    }, n


# --------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    rank, world, local_rank = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from rank_latent_attention_mixer_b200 import binding as fb
    from rank_latent_attention_mixer_b200 import workloads as W

    w = W.WORKLOADS[args.workload]
    w = w.with_shape(seed=rank_seed(w.seed, rank))
    if args.tokens:
        w = w.with_shape(N=args.tokens, name=f"{w.name}_n{args.tokens}")
    x = W.make_inputs(w, device=str(dev))
    if args.layout == "bnhd":
        for name in ("k0", "k", "v"):
            x[name] = x[name].transpose(1, 2).contiguous()
    path = {"auto": fb.PATH_AUTO, "simt": fb.PATH_SIMT, "tcgen05": fb.PATH_TCGEN05}[args.path]
    dtype_code = {"f32": fb.F32, "bf16": fb.BF16, "f16": fb.F16}[w.dtype]
    used_path = path or fb.selected_path(w.B, w.H, w.N, w.M, w.D, dtype_code)
    gated = not args.flare
    ws = torch.empty(fb.workspace_bytes(w.B, w.H, w.N, w.M, w.D, dtype_code, gated, path, layout=args.layout,
                                        norm_synthesis=args.norm), dtype=torch.uint8, device=dev)
    y = torch.empty_like(x["k"])
    norm = args.norm and gated
    n_launch = fb.launches_per_call(gated) + (1 if norm else 0)
    stage_names = (["rms_norm(q0, k0)"] if norm else []) + (STAGES_GATED if gated else STAGES_FLARE)
    fits_l2 = 5 * x["k"].numel() * x["k"].element_size() < L2_BYTES * 4
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev) if fits_l2 else None

    def step(events=None):
        fb.mixer_fwd(x["q0"], x["q_fixed"], x["gate"] if gated else None, x["k0"], x["k"], x["v"], y, path=path,
                     workspace=ws, stage_events=events, layout=args.layout, norm_synthesis=args.norm)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize()
    assert fb.check_device_status() == 0

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)] for _ in range(K)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            step(evs[i])
            if flush is not None:
                flush.zero_()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    status = fb.check_device_status()
    if status != 0:
        raise SystemExit(f"device status {status} after the timed region")

    stage_ms = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(n_launch)] for i in range(K)]
    if flush is None:
        local_ms = evs[0][0].elapsed_time(evs[K - 1][n_launch])
    else:
        local_ms = sum(evs[i][0].elapsed_time(evs[i][n_launch]) for i in range(K))
    max_ms = reduce_max(local_ms, world, dev)
    counts = W.algorithmic_counts(w, flare=not gated)
    value = aggregate_mtokens(counts["tokens"], world, K, max_ms)
    ms_per_step = max_ms / K

    # live per-kernel figures (this rank)
    avg_stage = [statistics.mean(s[j] for s in stage_ms) for j in range(n_launch)]
    total_stage = sum(avg_stage)
    stages = {stage_names[j]: {"ms": round(avg_stage[j], 4), "share": round(avg_stage[j] / total_stage, 4)}
              for j in range(n_launch)}
    o = 1 if norm else 0                   # the normalisation launch comes first
    split_ms = statistics.mean([avg_stage[o], avg_stage[o + 2]]) if gated else avg_stage[0]
    bhnmd = w.B * w.H * w.N * w.M * w.D
    flops_per_split_launch = 4.0 * bhnmd
    peaks, peak_src = load_peaks()
    # The timed region is well under a second of back-to-back calls at the
    # sampled clock, so the denominator is the burst GEMM peak (the sustained
    # one, taken over seconds under the power cap, is reported beside it).
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_ts = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_b = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    clk = sampler.summary()
    # bytes: mean of the split launches (synthesis reads k0 once, encode reads k and v)
    bytes_per_split_launch = (1.5 if gated else 2.0) * w.B * w.H * w.N * w.D * (4 if w.dtype == "f32" else 2)
    achieved_t = flops_per_split_launch / (split_ms * 1e-3) / 1e12
    achieved_b = bytes_per_split_launch / (split_ms * 1e-3) / 1e9
    # the binding roof: tensor pipe when the launch's FLOP/byte is above the measured ridge, else HBM
    tensor_bound = flops_per_split_launch / bytes_per_split_launch > peak_t * 1e12 / (peak_b * 1e9)
    roofline = {
        "bound": "tensor" if tensor_bound else "hbm",
        "kernel": "split_partial" if used_path == fb.PATH_TCGEN05 else "split_partial_simt",
        "achieved": round(achieved_t if tensor_bound else achieved_b, 2),
        "peak": peak_t if tensor_bound else peak_b,
        "unit": "TFLOP/s" if tensor_bound else "GB/s",
        "frac": round(achieved_t / peak_t if tensor_bound else achieved_b / peak_b, 4),
        "traffic": ncu_traffic("split_partial", w.name),
        "peak_kind": (f"{peak_src} bf16 burst (cuBLAS 8192^3, best of 10)"
                      + (" x 1 (dense fp16 runs at the bf16 rate)" if w.dtype == "f16" else "") if tensor_bound
                      else f"{peak_src} HBM copy bandwidth"),
        "frac_of_sustained": round(achieved_t / peak_ts, 4) if tensor_bound else None,
        "peak_sustained": peak_ts,
        # the achieved rate at the maximum SM clock: how much of the gap to the
        # peak is the clock the box ran at during the timed region
        "clock_scaled_frac": (round(achieved_t / peak_t * clk["sm_max_mhz"] / clk["sm_mhz"], 4)
                              if tensor_bound and clk.get("sm_mhz") and clk.get("sm_max_mhz") else None),
        "algorithmic_per_launch": {"flops": flops_per_split_launch, "bytes": bytes_per_split_launch},
        "launch_ms": round(split_ms, 4),
        "tensor_frac": round(achieved_t / peak_t, 4),
        "hbm_frac": round(achieved_b / peak_b, 4),
    }
    decode_ms = avg_stage[n_launch - 1]
    dec_t = 4.0 * bhnmd / (decode_ms * 1e-3) / 1e12

    out = {
        "metric": METRIC,
        "value": round(value, 4),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "M": w.M, "D": w.D, "io_dtype": w.dtype,
                   "gate": "open (FLARE++)" if gated else "closed (FLARE, flare_fwd)",
                   "layout": args.layout,
                   "synthesis_norm": bool(args.norm),
                   "kernel_path": {1: "simt", 2: "tcgen05"}.get(used_path, used_path),
                   "l2": ("flushed between steps (512 MiB write)" if flush is not None
                          else "inputs larger than L2 (back-to-back steps)"),
                   "parallelism": f"replicas x{world} (independent problems per rank)",
                   "seed_rank0": W.WORKLOADS[args.workload].seed},
        "tflops": round(counts["flops"] / (ms_per_step * 1e-3) / 1e12 * world, 2),
        "hbm_gbs_algorithmic": round(counts["bytes"] / (ms_per_step * 1e-3) / 1e9 * world, 1),
        "gpu_launches": K * n_launch,
        "roofline": roofline,
        "stages": stages,
        "decode": {"tflops": round(dec_t, 2), "frac_of_peak": round(dec_t / peak_t, 4)},
        "clocks": clk,
    }

    # back-to-back calls (no L2 flush, no per-launch events between them): the
    # launch sequence as a model calling the mixer layer after layer sees it,
    # with consecutive kernels overlapping set-up and tail (programmatic
    # dependent launch)
    kb = max(1, min(K, 30))
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    b0.record()
    for _ in range(kb):
        step()
    b1.record()
    torch.cuda.synchronize()
    b2b_ms = reduce_max(b0.elapsed_time(b1), world, dev) / kb
    out["back_to_back"] = {"ms_per_call": round(b2b_ms, 4), "calls": kb,
                           "value": round(aggregate_mtokens(counts["tokens"], world, 1, b2b_ms), 4), "unit": UNIT,
                           "l2": "not flushed between calls"}

    # end-to-end through the public API with host buffers
    if not args.no_e2e:
        hx = {}
        for name in ("q0", "q_fixed", "gate", "k0", "k", "v"):
            src = x[name].transpose(1, 2) if args.layout == "bnhd" and name in ("k0", "k", "v") else x[name]
            hx[name] = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
            hx[name].copy_(src)
        hy = torch.empty(hx["k"].shape, dtype=y.dtype, pin_memory=True)
        ke = max(1, min(K, 5))
        hg = hx["gate"] if gated else None
        fb.mixer_fwd_host(hx["q0"], hx["q_fixed"], hg, hx["k0"], hx["k"], hx["v"], hy)  # warm-up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(ke):
            fb.mixer_fwd_host(hx["q0"], hx["q_fixed"], hg, hx["k0"], hx["k"], hx["v"], hy)
        e1.record()
        torch.cuda.synchronize()
        e2e_ms = reduce_max(e0.elapsed_time(e1), world, dev)
        h2d = sum(hx[n].numel() * hx[n].element_size() for n in hx
                  if gated or n in ("q_fixed", "k", "v"))
        out["e2e"] = {"value": round(aggregate_mtokens(counts["tokens"], world, ke, e2e_ms), 4), "unit": UNIT,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hy.numel() * hy.element_size(),
                      "steps": ke, "api": "flarepp_mixer_fwd_host (pinned host buffers, [B,H,N,D])"}
        del hx, hy

    if (rank == 0 and world == 1 and not args.no_configs and not args.tokens and args.layout == "bhnd"
            and gated and not args.norm and args.path == "auto"):
        out["configs"] = config_records(fb, W, dev, peaks, peak_src, main=(w, x, y, ms_per_step, path))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb, _ = cpu_baseline(x, w, args.cpu_seconds)
        out["cpu_baseline"] = cb
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# --------------------------------------------------------------------------- every configuration

CONFIG_ORDER = [("tiny_f32", False), ("grid85_bf16", False), ("grid85_bf16", True), ("grid129_peaky_bf16", False),
                ("cloud40k_bf16", False), ("scale1m_bf16", False)]
TOL = {"f32": None, "bf16": (1e-2, 2e-2), "f16": (2.5e-3, 5e-3)}


def parity_figures(g, o, dtype):
    """Worst-case figures of one output against the fp64 oracle, with the bound."""
    import numpy as np
    g = g.detach().to("cpu", dtype=__import__("torch").float64).numpy() if hasattr(g, "detach") else np.asarray(g)
    o = np.asarray(o, dtype=np.float64)
    d = np.abs(g - o)
    rel_l2 = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-300))
    max_abs = float(d.max())
    if dtype == "f32":
        rows = d.reshape(-1, d.shape[-1]).max(axis=1) / np.maximum(np.abs(o).reshape(-1, d.shape[-1]).max(axis=1), 1e-30)
        worst = float(rows.max())
        return {"row_max_rel": worst, "bound": 1e-4, "pass": worst <= 1e-4}
    l2, ab = TOL[dtype]
    return {"rel_l2": rel_l2, "max_abs": max_abs, "bound": [l2, ab], "pass": rel_l2 <= l2 and max_abs <= ab}


def config_records(fb, W, dev, peaks, peak_src, main):
    """Every BASELINE workload (and the 7,225-token grid with the gate closed)
    timed on this GPU -- device time per call with the L2 flushed between calls
    -- with its binding roofline and its parity against the fp64 oracle: the
    whole outputs for the four small workloads, one head (q, z) and 256
    sampled tokens (y) for the 1M-token one (the test suite compares it in
    full)."""
    import numpy as np
    import torch
    import oracle
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_b = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    recs = {}
    for name, flare in CONFIG_ORDER:
        key = name + ("_gate0" if flare else "")
        wc = W.WORKLOADS[name]
        if name == main[0].name:
            xc, yc, ms, path = main[1], main[2], main[3], main[4]
        else:
            xc = W.make_inputs(wc, device=str(dev))
            yc = torch.empty_like(xc["k"])
            path = 0
            gate = None if flare else xc["gate"]
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            times = []
            for i in range(23):
                flush.zero_()
                ev[0].record()
                fb.mixer_fwd(xc["q0"], xc["q_fixed"], gate, xc["k0"], xc["k"], xc["v"], yc)
                ev[1].record()
                torch.cuda.synchronize()
                if i >= 3:
                    times.append(ev[0].elapsed_time(ev[1]))
            ms = statistics.median(times)
        counts = W.algorithmic_counts(wc, flare=flare)
        tfs = counts["flops"] / (ms * 1e-3) / 1e12
        gbs = counts["bytes"] / (ms * 1e-3) / 1e9
        tensor = counts["flops"] / counts["bytes"] > peak_t * 1e12 / (peak_b * 1e9) and wc.dtype != "f32"
        rec = {"B": wc.B, "H": wc.H, "N": wc.N, "M": wc.M, "D": wc.D, "dtype": wc.dtype,
               "gate": "closed (flare_fwd form)" if flare else "open",
               "ms_per_call": round(ms, 4), "mtokens_s": round(counts["tokens"] / (ms * 1e-3) / 1e6, 3),
               "tflops": round(tfs, 2), "gbs": round(gbs, 1),
               "bound": "tensor" if tensor else "hbm",
               "frac": round(tfs / peak_t if tensor else gbs / peak_b, 4),
               "peak": peak_t if tensor else peak_b, "peak_kind": f"{peak_src} " + ("bf16 burst" if tensor else "HBM"),
               "timing": "median of 20 calls, 512 MiB L2 flush before each" if name != main[0].name
                         else "the main line's steps"}
        # parity against the fp64 oracle
        if name.startswith("scale1m"):
            h = 5
            toks = np.random.default_rng(1).integers(0, wc.N, 256)
            toks[:2] = [0, wc.N - 1]
            yq, q, z = fb.mixer_fwd(xc["q0"], xc["q_fixed"], xc["gate"], xc["k0"], xc["k"], xc["v"],
                                    return_qz=True)
            torch.cuda.synchronize()
            y_ref, q_ref, z_ref = oracle.flarepp_head(xc["q0"][h], xc["q_fixed"][h], float(xc["gate"][h]),
                                                      xc["k0"][0, h], xc["k"][0, h], xc["v"][0, h], toks)
            rec["parity"] = {"sample": "head 5: q, z in full; y at 256 sampled tokens",
                             "y": parity_figures(yq[0, h, torch.from_numpy(toks).to(dev)], y_ref, wc.dtype),
                             "q": parity_figures(q[0, h], q_ref, wc.dtype),
                             "z": parity_figures(z[0, h], z_ref, wc.dtype)}
        else:
            xh = {k: v.cpu() for k, v in xc.items()}
            y_ref, q_ref, z_ref = oracle.flarepp(xh["q0"], xh["q_fixed"], None if flare else xh["gate"], xh["k0"],
                                                 xh["k"], xh["v"], flare=flare)
            rec["parity"] = {"sample": "whole outputs", "y": parity_figures(yc, y_ref, wc.dtype)}
        rec["parity"]["pass"] = all(v["pass"] for k, v in rec["parity"].items() if isinstance(v, dict))
        recs[key] = rec
        del xc, yc
        torch.cuda.empty_cache()
    return recs


# --------------------------------------------------------------------------- reference arm (the oracle)

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return  # rank 0 alone runs the CPU reference
    import torch
    from rank_latent_attention_mixer_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if w.device_rng:
        # The CPU generator takes minutes for 2.7 G numbers; the sample needs
        # one head, so draw that slice with the same recipe on the CPU.
        x = _cpu_head_inputs(w)
    else:
        x = W.make_inputs(w)
    budget = min(15.0, 150.0 / max(1, args.steps + args.warmup))
    head = head_slice_cpu(x, w)
    n_avail = head[3].shape[0]
    n_cal = min(n_avail, 1024)
    per_tok = max(oracle_sample(head, w, n_cal) / n_cal, 1e-9)
    n = int(min(n_avail, max(n_cal, budget / per_tok)))
    for _ in range(args.warmup):
        oracle_sample(head, w, n)
    times = [oracle_sample(head, w, n) for _ in range(args.steps)]
    t = statistics.mean(times)
    value = n / (t * w.H) / 1e6
    import oracle
    sample = (f"{w.name}: batch 0, head 0 of {w.H}, first {n} of {w.N} tokens, M={w.M}, D={w.D}, fp64 oracle; "
              f"tokens/s = sample tokens / (time x {w.H} heads)")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "M": w.M, "D": w.D},
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": oracle.num_threads(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def _cpu_head_inputs(w):
    """Head-0 slice of a device-drawn workload, drawn on the CPU with the same
    recipe (used only when no GPU runs: the reference arm)."""
    import torch
    from rank_latent_attention_mixer_b200 import workloads as W
    n = min(w.N, 262144)
    small = W.Workload(w.name + "_head0", 1, 1, n, w.M, w.D, w.dtype, w.seed, w.recipe, w.rms_q0, w.rms_k0)
    return W.make_inputs(small)


# --------------------------------------------------------------------------- token-sharded arm

def run_cp(args):
    """One global problem with its tokens sharded over the ranks: each rank
    runs the split passes on its N/world tokens, the latent-sized triples are
    all-gathered over NCCL and merged, and each rank decodes its tokens
    (strong scaling: total work fixed as the rank count grows)."""
    import torch
    rank, world, local_rank = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from rank_latent_attention_mixer_b200 import binding as fb
    from rank_latent_attention_mixer_b200 import cp
    from rank_latent_attention_mixer_b200 import workloads as W

    w = W.WORKLOADS[args.workload]                  # the same global problem on every rank
    if args.tokens:
        w = w.with_shape(N=args.tokens, name=f"{w.name}_n{args.tokens}")
    x = W.make_inputs(w, device=str(dev))
    lo, hi = cp.shard_bounds(w.N, world, rank)
    for name in ("k0", "k", "v"):
        t = x[name][:, :, lo:hi]
        x[name] = (t.transpose(1, 2) if args.layout == "bnhd" else t).contiguous()
    torch.cuda.empty_cache()
    n_local = hi - lo
    path = {"auto": fb.PATH_AUTO, "simt": fb.PATH_SIMT, "tcgen05": fb.PATH_TCGEN05}[args.path]
    gated = not args.flare
    y = torch.empty_like(x["k"])
    fits_l2 = 5 * x["k"].numel() * x["k"].element_size() < L2_BYTES * 4
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev) if fits_l2 else None

    class TimedOps:
        """The library stages, with events around each split pass on the launching stream."""
        def __init__(self):
            self.marks = None

        def __getattr__(self, name):
            return getattr(fb, name)

        def cp_partials(self, *a, **kw):
            if self.marks is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fb.cp_partials(*a, **kw)
                e1.record()
                self.marks.append((e0, e1))
            else:
                fb.cp_partials(*a, **kw)

    ops = TimedOps()

    if args.backward:
        dy = W.random_cotangent((w.B, w.H, w.N, w.D), w.dtype, seed=w.seed + 100, device=str(dev),
                                device_rng=w.device_rng)[:, :, lo:hi]
        dy = (dy.transpose(1, 2) if args.layout == "bnhd" else dy).contiguous()

    def step():
        if args.backward:
            cp.mixer_bwd_cp(x["q0"], x["q_fixed"], x["gate"] if gated else None, x["k0"], x["k"], x["v"], dy,
                            layout=args.layout, path=path, _ops=ops)
        else:
            cp.mixer_fwd_cp(x["q0"], x["q_fixed"], x["gate"] if gated else None, x["k0"], x["k"], x["v"], y,
                            layout=args.layout, path=path, _ops=ops)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize()
    assert fb.check_device_status() == 0
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    ops.marks = []
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            ev[i][0].record()
            step()
            ev[i][1].record()
            if flush is not None:
                flush.zero_()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    if fb.check_device_status() != 0:
        raise SystemExit("device status after the timed region")
    local_ms = sum(a.elapsed_time(b) for a, b in ev)
    max_ms = reduce_max(local_ms, world, dev)
    split_ms = statistics.mean(a.elapsed_time(b) for a, b in ops.marks)
    counts = W.algorithmic_counts(w, flare=not gated)
    value = counts["tokens"] * K / (max_ms * 1e-3) / 1e6          # the global problem's tokens
    peaks, peak_src = load_peaks()
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    flops_split = 4.0 * w.B * w.H * n_local * w.M * w.D
    achieved = flops_split / (split_ms * 1e-3) / 1e12
    out = {
        "metric": ("FLARE++ mixer bwd Mtokens/s (token-sharded)" if args.backward else METRIC),
        "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(max_ms / K, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "M": w.M, "D": w.D, "io_dtype": w.dtype,
                   "gate": "open (FLARE++)" if gated else "closed (FLARE)", "layout": args.layout,
                   "parallelism": f"token-sharded x{world} ({n_local} tokens on rank {rank}; NCCL all-gather of "
                                  f"latent triples)",
                   "l2": ("flushed between steps (512 MiB write)" if flush is not None
                          else "inputs larger than L2 (back-to-back steps)")},
        "tflops": round(counts["flops"] / (max_ms / K * 1e-3) / 1e12, 2),
        # forward: split + triple merge per sharded pass, merges, decode (+1 normalisation);
        # backward: the recomputed sharded passes and merges, then stages 1-4 (3, 4, 4 and 2
        # launches gated; 3, 4, 1, 1 closed)
        "gpu_launches": K * (((6 if gated else 3) + (13 if gated else 9)) if args.backward
                             else ((5 if gated else 3) + (2 if gated else 1))),
        "roofline": {"bound": "tensor", "kernel": "split_partial (+ local triple reduction)",
                     "achieved": round(achieved, 2), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_t, 4), "traffic": None,
                     "peak_kind": f"{peak_src} bf16 burst", "launch_ms": round(split_ms, 4)},
        "clocks": sampler.summary(),
    }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# --------------------------------------------------------------------------- backward arm

BWD_STAGES_GATED = ["fwd split(synthesis)", "fwd merge(q)", "fwd split(encode)", "fwd merge(z)",
                    "decode_rows", "decode_cols", "reduce(decode)", "token_cols(encode)", "latent_rows(encode)",
                    "reduce(encode)", "token_cols(synthesis)", "latent_rows(synthesis)", "reduce(synthesis)",
                    "reduce_batch"]
BWD_STAGES_FLARE = ["fwd split(encode)", "fwd merge(z)", "decode_rows", "decode_cols", "reduce(decode)",
                    "token_cols(encode)", "latent_rows(encode)", "reduce(encode)", "reduce_batch"]
BWD_TC_STAGES_GATED = ["fwd split(synthesis)", "fwd merge(q)", "fwd split(encode)", "fwd merge(z)",
                       "fwd decode(stats)", "tc_latent(decode)", "reduce(decode)", "tc_token(decode+encode)",
                       "tc_latent(encode)", "reduce(encode)", "tc_token(synthesis)", "tc_latent(synthesis)",
                       "reduce(synthesis)", "reduce_batch"]
BWD_TC_STAGES_FLARE = ["fwd split(encode)", "fwd merge(z)", "fwd decode(stats)", "tc_latent(decode)",
                       "reduce(decode)", "tc_token(decode+encode)", "tc_latent(encode)", "reduce(encode)",
                       "reduce_batch"]
# FLOPs per (b, h, n, m, d) of each backward kernel as executed (2 per multiply-add):
# decode rows recompute the decode softmax and y (4), then score, <dy, z> and dS q (6)
BWD_KERNEL_FLOPS = {"decode_rows": 10, "decode_cols": 8, "token_cols": 8, "latent_rows": 6}
# tensor-core kernel: S and dP (4; the fused token side has two dP: 6), acc1 (2), acc2 (2 where present)
BWD_TC_FLOPS = {"tc_latent(decode)": 8, "tc_token(decode+encode)": 10, "tc_latent(encode)": 6,
                "tc_token(synthesis)": 8, "tc_latent(synthesis)": 6}


def fp32_simt_peak_tflops(peaks):
    """FP32 FMA peak of the SIMT pipes: 148 SMs x 128 lanes x 2 FLOP per clock
    at the maximum SM clock."""
    mhz = peaks.get("sm_max_mhz", 1965.0)
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def run_backward_bench(args):
    import torch
    rank, world, local_rank = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from rank_latent_attention_mixer_b200 import binding as fb
    from rank_latent_attention_mixer_b200 import workloads as W

    w = W.WORKLOADS[args.workload]
    w = w.with_shape(seed=rank_seed(w.seed, rank))
    if args.tokens:
        w = w.with_shape(N=args.tokens, name=f"{w.name}_n{args.tokens}")
    x = W.make_inputs(w, device=str(dev))
    dy = W.random_cotangent((w.B, w.H, w.N, w.D), w.dtype, seed=w.seed + 100, device=str(dev),
                            device_rng=w.device_rng)
    path = {"auto": fb.PATH_AUTO, "simt": fb.PATH_SIMT, "tcgen05": fb.PATH_TCGEN05}[args.path]
    dtype_code = {"f32": fb.F32, "bf16": fb.BF16, "f16": fb.F16}[w.dtype]
    gated = not args.flare
    norm = args.norm and gated
    ws = torch.empty(fb.bwd_workspace_bytes(w.B, w.H, w.N, w.M, w.D, dtype_code, path, norm_synthesis=norm),
                     dtype=torch.uint8, device=dev)
    out_t = {"dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"]),
             "dq_fixed": torch.empty((w.H, w.M, w.D), dtype=torch.float32, device=dev)}
    if gated:
        out_t.update(dk0=torch.empty_like(x["k0"]), dq0=torch.empty((w.H, w.M, w.D), dtype=torch.float32, device=dev),
                     dgate=torch.empty((w.H,), dtype=torch.float32, device=dev))
    used_path = path or fb.selected_path(w.B, w.H, w.N, w.M, w.D, dtype_code)
    if used_path == fb.PATH_TCGEN05:
        names = BWD_TC_STAGES_GATED if gated else BWD_TC_STAGES_FLARE
    else:
        names = BWD_STAGES_GATED if gated else BWD_STAGES_FLARE
    extra_kernels = 0
    saved = None
    if args.saved_state:
        # the recomputed forward passes are replaced by the saved state
        names = [nm for nm in names if not nm.startswith("fwd ")]
        if used_path == fb.PATH_TCGEN05:
            names = ["round(q, z)", "token <dy, y>"] + names
            extra_kernels = 1                      # the rounding stage is two launches
        y_fwd, ctx = fb.mixer_fwd_train(x["q0"], x["q_fixed"], x["gate"] if gated else None, x["k0"], x["k"],
                                        x["v"], path=path, norm_synthesis=norm)
        saved = (y_fwd, ctx)
    if norm:
        names = ["rms_norm(q0, k0)"] + names + ["rms_bwd(k0)", "rms_bwd(q0)"]
    n_launch = len(names)
    fits_l2 = 6 * x["k"].numel() * x["k"].element_size() < L2_BYTES * 4
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev) if fits_l2 else None

    def step(events=None):
        fb.mixer_bwd(x["q0"], x["q_fixed"], x["gate"] if gated else None, x["k0"], x["k"], x["v"], dy, path=path,
                     workspace=ws, stage_events=events, out=out_t, norm_synthesis=norm,
                     ctx=saved[1] if saved else None, y=saved[0] if saved else None)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize()
    assert fb.check_device_status() == 0
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)] for _ in range(K)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            step(evs[i])
            if flush is not None:
                flush.zero_()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    if fb.check_device_status() != 0:
        raise SystemExit("device status after the timed region")
    local_ms = sum(evs[i][0].elapsed_time(evs[i][n_launch]) for i in range(K))
    max_ms = reduce_max(local_ms, world, dev)
    stage = [statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) for j in range(n_launch)]
    total = sum(stage)
    bhnmd = w.B * w.H * w.N * w.M * w.D
    peaks, peak_src = load_peaks()
    peak_alu = fp32_simt_peak_tflops(peaks)
    kern = {}
    tc_path = used_path == fb.PATH_TCGEN05

    def flops_of(nm):
        return BWD_TC_FLOPS.get(nm) if tc_path else BWD_KERNEL_FLOPS.get(nm.split("(")[0])

    for nm, ms in zip(names, stage):
        f = flops_of(nm)
        kern[nm] = {"ms": round(ms, 4), "share": round(ms / total, 4)}
        if f:
            kern[nm]["tflops"] = round(f * bhnmd / (ms * 1e-3) / 1e12, 2)
    # the dominant backward kernel's roofline: the tensor pipe (tcgen05 kernel) or
    # SIMT fp32 FMA arithmetic
    top = max((nm for nm in names if flops_of(nm)), key=lambda nm: kern[nm]["ms"])
    achieved = kern[top]["tflops"]
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_ts = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    counts = W.algorithmic_counts(w, flare=not gated)
    ms_step = max_ms / K
    passes = 3 if gated else 2
    out = {
        "metric": "FLARE++ mixer bwd Mtokens/s on 1 B200 (gradients of every input)",
        "value": round(aggregate_mtokens(counts["tokens"], world, K, max_ms), 4), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "M": w.M, "D": w.D, "io_dtype": w.dtype,
                   "gate": "open (FLARE++)" if gated else "closed (FLARE)", "synthesis_norm": norm,
                   "saved_state": bool(args.saved_state),
                   "kernel_path": {1: "simt", 2: "tcgen05"}.get(used_path, used_path),
                   "l2": ("flushed between steps (512 MiB write)" if flush is not None
                          else "inputs larger than L2 (back-to-back steps)")},
        "algorithmic_tflops": round(10.0 * passes * bhnmd / (ms_step * 1e-3) / 1e12, 2),
        "gpu_launches": K * (n_launch + extra_kernels),
        "roofline": ({"bound": "tensor", "kernel": top, "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                      "frac": round(achieved / peak_t, 4), "traffic": None,
                      "frac_of_sustained": round(achieved / peak_ts, 4),
                      "peak_kind": f"{peak_src} bf16 burst"} if tc_path else
                     {"bound": "alu", "kernel": top, "achieved": achieved, "peak": round(peak_alu, 1),
                      "unit": "TFLOP/s", "frac": round(achieved / peak_alu, 4), "traffic": None,
                      "peak_kind": "FP32 FMA: 148 SMs x 128 lanes x 2 FLOP x max SM clock"}),
        "stages": kern,
        "clocks": sampler.summary(),
    }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    elif args.cp:
        run_cp(args)
    elif args.backward:
        run_backward_bench(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
