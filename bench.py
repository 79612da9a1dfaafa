#!/usr/bin/env python
"""Benchmark of the MoE layer hot path (plan -> dispatch -> grouped SwiGLU FFN -> combine).

One step = one full layer call (all micro-batches of the workload) through the C ABI
(moe_forward) with inputs resident in HBM. Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload deepseek_v3]
  python bench.py --impl reference ...      # the CPU oracle, timed on the host cores

Multi-GPU (torchrun, one process per GPU): every rank runs an independent replica of
the layer on its own tokens (the layer has no exchange step on one GPU: replicas only);
value = tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402

METRIC = ("MoE layer tokens/sec on 1 B200; dispatch+combine HBM GB/s; "
          "grouped-GEMM % bf16 peak")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["moe", "reference"], default="moe")
    ap.add_argument("--workload", default="deepseek_v3")
    ap.add_argument("--streaming", type=int, default=-1,
                    help="1: FFN claims tiles while dispatch runs; 0: serial; -1: default")
    ap.add_argument("--packed", type=int, default=1,
                    help="1: prepack the weights once before timing (moe_pack_weights)")
    ap.add_argument("--ffn-kernel", type=int, default=0,
                    help="grouped-GEMM kernel: 1 one CTA per unit, 2 SM pairs; 0: default")
    ap.add_argument("--early-combine", type=int, default=-1,
                    help="1: combine fused into GEMM Y (early combine); 0: separate combine; "
                         "-1: default")
    ap.add_argument("--ab", type=int, default=1,
                    help="1: also time early combine and streaming against the timed "
                         "configuration, alternating on this GPU (reported under 'ab')")
    ap.add_argument("--backward", type=int, default=1,
                    help="1: also time moe_backward (after one forward), reported under 'backward'")
    ap.add_argument("--ep", type=int, default=8,
                    help="expert-parallel ranks emulated on this GPU for the 'ep' section "
                         "(0: skip; needs E and T divisible by it)")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=16, help="oracle tokens per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ environment helpers

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, \
            "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def reduce_max(values, device, world):
    """Element-wise max over ranks (all_reduce MAX); identity for one rank."""
    import torch
    if world == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tokens_per_s(world, tokens_per_step, ms_per_step):
    """All ranks' tokens per step over the slowest rank's time per step."""
    return world * tokens_per_step / (ms_per_step / 1000.0)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while the timed region runs."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def mark(self, begin: bool):
        """Host wall time of the start / end of the timed region (samples outside are dropped)."""
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.idx)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            if ts is not None and self.t0 is not None and not (self.t0 <= ts <= self.t1):
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, parts[5:9]):
                if val.lower() in ("active", "1"):
                    reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(power) if power else None}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


KERNEL_SOURCES = {
    "ffn_gemm_kernel<0>": ("ffn_gemm.cu", "ffn_gemm.cuh", "moe_common.cuh", "moe_internal.h"),
    "ffn_gemm_kernel<1>": ("ffn_gemm.cu", "ffn_gemm.cuh", "moe_common.cuh", "moe_internal.h"),
    "ffn_gemm_pair_kernel<0>": ("ffn_gemm_pair.cu", "ffn_gemm.cuh", "moe_common.cuh",
                                "moe_internal.h"),
    "ffn_gemm_pair_kernel<1>": ("ffn_gemm_pair.cu", "ffn_gemm.cuh", "moe_common.cuh",
                                "moe_internal.h"),
    "dispatch_kernel": ("dispatch.cu", "moe_common.cuh", "moe_internal.h"),
}


def kernel_source_hash(kernel: str = "ffn_gemm_kernel<0>") -> str:
    """Hash of the source files a kernel is built from (its committed counters are only
    used while this matches)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "combine_moe_plan_03_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu summary, if it
    was taken on that workload and on the current kernel sources (else None: no capture,
    or the counters are stale)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    ent = d.get(kernel)
    if (not ent or ent.get("source_hash") != kernel_source_hash(kernel)
            or ent.get("workload") != workload):
        return None
    return ent.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ inputs

def host_weights(cfg):
    """Full W1 / W2 on the host (bf16 bit patterns)."""
    return si.make_w1(cfg), (si.make_w2(cfg) if cfg.I > 0 else None)


def upload_weights(cfg, dev, rank, world, keep_host: bool):
    """Rank 0 generates the weights and copies them to its GPU; other ranks receive them by
    broadcast (setup only, outside the timed region)."""
    import torch
    W1 = torch.empty((cfg.E, cfg.H, 2 * cfg.I), dtype=torch.bfloat16, device=dev)
    W2 = torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16, device=dev)
    host = None
    if rank == 0:
        if keep_host:
            h1, h2 = host_weights(cfg)
            W1.copy_(torch.from_numpy(h1.view(np.int16)).view(torch.bfloat16))
            W2.copy_(torch.from_numpy(h2.view(np.int16)).view(torch.bfloat16))
            host = (h1, h2)
        else:
            n1 = cfg.H * 2 * cfg.I
            n2 = cfg.I * cfg.H
            for e in range(cfg.E):
                h1 = si.normal_bf16(cfg.seed, si.STREAM_W1, e * n1, n1, cfg.w1_sigma())
                W1[e].copy_(torch.from_numpy(h1.view(np.int16)).view(torch.bfloat16)
                            .view(cfg.H, 2 * cfg.I))
                h2 = si.normal_bf16(cfg.seed, si.STREAM_W2, e * n2, n2, cfg.w2_sigma())
                W2[e].copy_(torch.from_numpy(h2.view(np.int16)).view(torch.bfloat16)
                            .view(cfg.I, cfg.H))
    if world > 1:
        import torch.distributed as dist
        dist.broadcast(W1, src=0)
        dist.broadcast(W2, src=0)
    return W1, W2, host


# ------------------------------------------------------------------ CPU oracle timing

def oracle_tokens_per_s(cfg, x, idx, w, W1h, W2h, tokens, threads):
    import oracle
    orc = oracle.get()
    W1l = [W1h[e] for e in range(cfg.E)]
    W2l = [W2h[e] for e in range(cfg.E)]
    t0 = time.perf_counter()
    orc.moe_forward(x[tokens], idx[tokens], w[tokens], W1l, W2l, n_threads=threads)
    return len(tokens) / (time.perf_counter() - t0)


def cpu_baseline(cfg, x, idx, w, host, budget_s):
    """The oracle as it stands on the host cores, on a bounded sample of the workload's tokens."""
    threads = os.cpu_count() or 1
    W1h, W2h = host
    rng = np.random.default_rng(0)
    probe = np.sort(rng.choice(cfg.T, size=min(cfg.T, threads), replace=False))
    rate = oracle_tokens_per_s(cfg, x, idx, w, W1h, W2h, probe, threads)
    n = int(max(threads, min(cfg.T, rate * budget_s)))
    n = (n // threads) * threads or threads
    sample = np.sort(rng.choice(cfg.T, size=min(n, cfg.T), replace=False))
    t0 = time.perf_counter()
    val = oracle_tokens_per_s(cfg, x, idx, w, W1h, W2h, sample, threads)
    return {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(sample)} of {cfg.T} tokens of {cfg.name} (seeded), "
                      f"{time.perf_counter() - t0:.1f} s, fp64 C oracle with OpenMP"}


def run_reference(args):
    """--impl reference: the CPU oracle timed on the host cores (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    cfg = si.CONFIGS[args.workload]
    threads = os.cpu_count() or 1
    orc = oracle.get()
    x = si.make_x(cfg)
    idx, w = si.make_routing(cfg)
    rng = np.random.default_rng(1)
    n = max(1, args.ref_tokens)
    cache1, cache2 = {}, {}

    def wts(tokens):
        need = sorted(set(int(e) for e in idx[tokens].reshape(-1) if e >= 0))
        for e in need:
            if e not in cache1:
                if cfg.identity:
                    continue
                cache1[e] = si.make_w1_expert(cfg, e)
                cache2[e] = si.make_w2_expert(cfg, e)
        return [cache1.get(e) for e in range(cfg.E)], [cache2.get(e) for e in range(cfg.E)]

    def step():
        tokens = np.sort(rng.choice(cfg.T, size=min(n, cfg.T), replace=False))
        if cfg.identity:
            t0 = time.perf_counter()
            orc.moe_forward_identity(x[tokens], idx[tokens], w[tokens])
            return len(tokens), time.perf_counter() - t0
        W1l, W2l = wts(tokens)
        t0 = time.perf_counter()
        orc.moe_forward(x[tokens], idx[tokens], w[tokens], W1l, W2l, n_threads=threads)
        return len(tokens), time.perf_counter() - t0

    for _ in range(args.warmup):
        step()
    tok = secs = 0.0
    for _ in range(args.steps):
        a, b = step()
        tok += a
        secs += b
    val = tok / secs
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, world),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle",
                             "sample": f"{n} tokens per step of {cfg.name}, {args.steps} steps"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_block(cfg, world):
    return {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
            "tile": cfg.tile, "micro_batches": cfg.micro_batches, "routing": cfg.routing,
            "identity_experts": cfg.identity,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2: each step streams the weights and pool (GBs) "
                  "through the 126 MB L2"}


# ------------------------------------------------------------------ the CUDA path

def tensor_peak(clocks: dict, timed_s: float, peaks: dict, peak_src: str):
    """The measured bf16 peak a tensor-bound kernel's roofline is taken against, chosen from
    the run's own clock record: the burst rate (a cuBLAS GEMM timed alone, at full clock)
    unless the timed region lasted seconds and the power cap held the median SM clock well
    below its maximum, as in the driver's seconds-long sustained cuBLAS loop.
    Returns (peak TFLOP/s, description)."""
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = ("sw_power_cap" in (clocks.get("reasons") or []) and sm and smax
              and sm < 0.9 * smax and timed_s >= 2.0)
    if capped:
        return peaks["bf16_tflops_sustained"], (
            f"{peak_src} bf16 sustained: {timed_s:.1f} s timed at a median {sm:.0f} of "
            f"{smax:.0f} MHz under sw_power_cap")
    return peaks["bf16_tflops"], (
        f"{peak_src} bf16 burst: {timed_s:.2f} s timed, median SM clock "
        f"{sm if sm is None else round(sm)} of {smax if smax is None else round(smax)} MHz")


def hbm_probe_rates(moe, dev, nbytes: int = 2 << 30, reps: int = 10):
    """Write-only and copy rates of this library's own probe kernels (moe_hbm_probe) on this
    GPU, CUDA events around `reps` launches over buffers far larger than L2: the ceilings that
    dispatch (mostly writes) and combine (mostly reads) are compared with. GB/s, copy counted
    as read + write bytes."""
    import torch
    half = nbytes // 2
    a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream(dev).cuda_stream
    out = {}
    for name, mode, dst, src, n, moved in (
            ("write_v4_gbs", 0, a.data_ptr(), 0, nbytes, nbytes),
            ("write_bulk_gbs", 1, a.data_ptr(), 0, nbytes, nbytes),
            ("copy_gbs", 2, a.data_ptr() + half, a.data_ptr(), half, 2 * half)):
        for _ in range(2):
            moe.moe_hbm_probe(dst, src, n, mode, st)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(reps):
            moe.moe_hbm_probe(dst, src, n, mode, st)
        s1.record()
        torch.cuda.synchronize()
        out[name] = moved * reps / (s0.elapsed_time(s1) / 1e3) / 1e9
    del a
    torch.cuda.empty_cache()
    return out


def copy_bound_ms(read_bytes: float, write_bytes: float, rates: dict) -> float:
    """Shortest time for a kernel that reads and writes these bytes at the probed rates: its
    writes alone at the best write-only rate, and all its bytes at the copy rate."""
    w = max(rates["write_v4_gbs"], rates["write_bulk_gbs"])
    return 1e3 * max(write_bytes / (w * 1e9), (read_bytes + write_bytes) / (rates["copy_gbs"] * 1e9))


def streams_weights(pairs: float, n_live_experts: float, peaks: dict) -> bool:
    """True when a grouped GEMM over these routed pairs is bound by streaming its weights
    from HBM rather than by the tensor pipe: it does 2 * rows flops per weight element
    (2 bytes), so the ridge is the sustained bf16 rate over the HBM copy rate."""
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    return pairs / max(n_live_experts, 1.0) < ridge


def ab_layer_ms(moe, buf, dx, didx, dw, W1, W2, variants: dict, rounds: int = 4,
                calls: int = 10) -> dict:
    """Layer time per call of each named moe_config, measured in alternating rounds of
    `calls` calls (CUDA events from the communicate stream's start to the compute stream's
    end), so that every variant sees the same clock and power state; the median round."""
    import torch
    mbs = len(dx)
    res = {k: [] for k in variants}
    for k, c in variants.items():                      # warm-up of each variant
        for m in range(mbs):
            buf.forward(dx[m], didx[m], dw[m], W1, W2, c)
    torch.cuda.synchronize()
    for _ in range(rounds):
        for k, c in variants.items():
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(buf.comm)
            for _ in range(calls):
                for m in range(mbs):
                    buf.forward(dx[m], didx[m], dw[m], W1, W2, c)
            s1.record(buf.compute)
            torch.cuda.synchronize()
            res[k].append(s0.elapsed_time(s1) / calls)
    code, aux = moe.moe_get_status(buf.plan)
    if code != 0:
        raise RuntimeError(f"device status after the A/B: {moe.moe_strerror(code)} ({aux})")
    return {k: statistics.median(v) for k, v in res.items()}


def time_backward(moe, buf, cfg, dev, world, local, x, idx, w, W1, W2, W1u, W2u, packed, pairs,
                  peaks, peak_src, steps):
    """A training step of the layer on micro-batch 0: the forward that also keeps the gate /
    up values (moe_config.gate_up) and the backward that reads them, each timed over
    `steps` calls back to back with per-phase CUDA events (max over ranks)."""
    import ctypes
    import torch
    H, I, T = cfg.H, cfg.I, cfg.T
    fwd_ev = moe.moe_timing_events_create(7 * steps)
    farr = [(ctypes.c_void_p * 7)(*fwd_ev[7 * c: 7 * c + 7]) for c in range(steps)]
    # the training step keeps g | u, which needs the SM-pair kernels (the default)
    fcfg = [moe.moe_config(0, 0, 0, packed, moe.MOE_FFN_SM_PAIR, ctypes.cast(a, ctypes.c_void_p))
            for a in farr]
    for _ in range(3):
        buf.forward(x, idx, w, W1, W2, moe.moe_config(0, 0, 0, packed, moe.MOE_FFN_SM_PAIR, None),
                    save_for_backward=True)
    torch.cuda.synchronize()
    barrier(world)
    for c in range(steps):
        buf.forward(x, idx, w, W1, W2, fcfg[c], save_for_backward=True)
    torch.cuda.synchronize()
    el = moe.moe_event_elapsed_ms
    fwd_ms = el(fwd_ev[0], fwd_ev[7 * (steps - 1) + 6]) / steps
    fwd_gemm_a = sum(el(fwd_ev[7 * c + 3], fwd_ev[7 * c + 4]) for c in range(steps)) / steps
    moe.moe_events_destroy(fwd_ev)
    dy = torch.from_numpy(si.make_dy(cfg).view(np.int16)).to(dev).view(torch.bfloat16)
    gx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    gw = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    gW1 = torch.empty((cfg.E, H, 2 * I), dtype=torch.bfloat16, device=dev)
    gW2 = torch.empty((cfg.E, I, H), dtype=torch.bfloat16, device=dev)
    plain = moe.moe_config(0, 0, 0, 0, 0, None)
    for _ in range(3):
        buf.backward(dy, w, W1u, W2u, plain, dx=gx, dw=gw, dW1=gW1, dW2=gW2)
    torch.cuda.synchronize()
    tev = moe.moe_timing_events_create(8 * steps)
    arrs = [(ctypes.c_void_p * 8)(*tev[8 * c: 8 * c + 8]) for c in range(steps)]
    cfgs = [moe.moe_config(0, 0, 0, 0, 0, ctypes.cast(a, ctypes.c_void_p)) for a in arrs]
    sampler = ClockSampler(physical_gpu_index(local))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    sampler.mark(True)
    t_wall = time.perf_counter()
    for c in range(steps):
        buf.backward(dy, w, W1u, W2u, cfgs[c], dx=gx, dw=gw, dW1=gW1, dW2=gW2)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    sampler.mark(False)
    clocks = sampler.stop()
    code, aux = moe.moe_get_status(buf.plan)
    if code != 0:
        raise RuntimeError(f"device status after the backward: {moe.moe_strerror(code)} ({aux})")
    names = ("combine_bwd", "recompute_gu", "gemm_y_bwd", "wgrad_w2", "gemm_a_bwd", "wgrad_w1",
             "dispatch_bwd")
    ph = {k: 0.0 for k in names}
    for c in range(steps):
        e = tev[8 * c: 8 * c + 8]
        for i, k in enumerate(names):
            ph[k] += el(e[i], e[i + 1]) / steps
    total = el(tev[0], tev[8 * (steps - 1) + 7]) / steps
    red = reduce_max([total, fwd_ms, fwd_gemm_a] + [ph[k] for k in names], dev, world)
    total, fwd_ms, fwd_gemm_a, ph = red[0], red[1], red[2], dict(zip(names, red[3:]))
    moe.moe_events_destroy(tev)
    flops_gemm = pairs * 6.0 * H * I            # backward Y 2HI + backward A 4HI (g, u kept)
    gemm_ms = ph["gemm_y_bwd"] + ph["gemm_a_bwd"]
    wg_bytes = cfg.E * 3.0 * H * I * 2          # dW1 + dW2 written (bf16)
    wg_ms = ph["wgrad_w1"] + ph["wgrad_w2"]
    a_tf = pairs * 4.0 * H * I / (ph["gemm_a_bwd"] / 1e3) / 1e12
    # backward A reads W1 K-major: 2*rows flops per weight element, as GEMM A; with fewer
    # live rows per expert than the ridge it streams W1 from HBM
    idx_h = idx.cpu().numpy()
    n_live = float(len(np.unique(idx_h[idx_h >= 0])))
    if not streams_weights(pairs, n_live, peaks):
        tpk, tsrc = tensor_peak(clocks, t_wall, peaks, peak_src)
        bwd_roofline = {"kernel": "ffn_gemm_pair_kernel<1, K-major W1> (backward A)",
                        "bound": "tensor", "achieved": a_tf, "peak": tpk, "unit": "TFLOP/s",
                        "frac": a_tf / tpk, "peak_source": tsrc,
                        "frac_of_burst": a_tf / peaks["bf16_tflops"],
                        "frac_of_sustained": a_tf / peaks["bf16_tflops_sustained"],
                        "algorithmic": "useful flops pairs*4*H*I per launch"}
    else:
        a_gbs = ((n_live * H * 2 * I * 2 + pairs * (2 * I + H) * 2)
                 / (ph["gemm_a_bwd"] / 1e3) / 1e9)
        bwd_roofline = {"kernel": "ffn_gemm_pair_kernel<1, K-major W1> (backward A)",
                        "bound": "hbm", "achieved": a_gbs, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": a_gbs / peaks["hbm_gbs"],
                        "peak_source": f"{peak_src} HBM copy",
                        "algorithmic": "bytes per launch: W1 of the live experts + live rows "
                                       "of d(g, u) read + of d(pool) written"}
    cb_bytes = T * H * 2 + 2 * pairs * H * 2 + T * cfg.k * 8
    db_bytes = pairs * H * 2 + T * H * 2
    # the backward's mirrored overlaps against the serial order, alternating on this GPU:
    # early dispatch backward (folded into backward A) and the streaming combine backward
    # (tile order on the communicate stream, backward Y taking tiles on the compute stream)
    overlap = None
    if world == 1:
        def bwd_ms(c_, n=3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(buf.compute)
            for _ in range(n):
                buf.backward(dy, w, W1u, W2u, c_, dx=gx, dw=gw, dW1=gW1, dW2=gW2)
            e1.record(buf.compute)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n
        variants = {"serial": moe.moe_config(), "early_dispatch_bwd": moe.moe_config(early_combine=1),
                    "streaming_combine_bwd": moe.moe_config(streaming=1),
                    "both": moe.moe_config(streaming=1, early_combine=1)}
        for c_ in variants.values():
            bwd_ms(c_, 1)
        acc = {k: [] for k in variants}
        for _ in range(3):
            for k_, c_ in variants.items():
                acc[k_].append(bwd_ms(c_))
        code, aux = moe.moe_get_status(buf.plan)
        if code != 0:
            raise RuntimeError(f"device status after the backward A/B: {moe.moe_strerror(code)}")
        overlap = {"ms_per_call": {k: float(np.median(v)) for k, v in acc.items()},
                   "note": "median of 3 alternating rounds of 3 calls each, with weight gradients"}
    return {"ms_per_call": total, "tokens_per_s": world * T / (total / 1e3),
            "overlap_ab": overlap,
            "train_step": {"forward_saving_gate_up_ms": fwd_ms,
                           "forward_gemm_a_ms": fwd_gemm_a, "backward_ms": total,
                           "ms": fwd_ms + total,
                           "tokens_per_s": world * T / ((fwd_ms + total) / 1e3)},
            "phases_ms_per_call": {k: round(v, 5) for k, v in ph.items()},
            "grouped_gemms_useful_tflops": flops_gemm / (gemm_ms / 1e3) / 1e12,
            "weight_grads": {"ms": wg_ms, "useful_tflops": flops_gemm / (wg_ms / 1e3) / 1e12,
                             "written_gbs": wg_bytes / (wg_ms / 1e3) / 1e9,
                             "note": "dW1 [E,H,2I] + dW2 [E,I,H] in bf16; the writes bound it"},
            "combine_bwd_gbs": cb_bytes / (ph["combine_bwd"] / 1e3) / 1e9,
            "dispatch_bwd_gbs": db_bytes / (ph["dispatch_bwd"] / 1e3) / 1e9,
            "roofline": bwd_roofline,
            "weights": "as given (read K-major by the backward GEMMs)",
            "calls": steps, "gpu_launches": 9 * steps, "clocks": clocks,
            "note": "after a forward that kept g | u (no recompute); every call computes the "
                    "same gradients"}


BUILT_LIBS = (os.path.join(ROOT, "combine_moe_plan_03_b200", "libmoe.so"),
              os.path.join(ROOT, "oracle", "liboracle.so"),
              os.path.join(ROOT, "synth_inputs", "libsynth.so"))


def time_ep(moe, cfg, dev, x, idx, w, W1, W2, packed, R, single_out, peaks, reps=10):
    """The expert-parallel layer (moe_ep_*) with R ranks emulated on this GPU: rank r takes
    tokens [r T/R, (r+1) T/R) of the workload and owns experts [r E/R, (r+1) E/R); every
    rank's buffers live here, so the "peer" stores and loads are local HBM traffic. One
    layer call = each rank's plan, the count exchange (a device copy standing in for the
    all-gather of E integers), each rank's layout, dispatch, grouped FFN and combine, all on
    one stream. Also reported: the bytes each rank would move over NVLink and the time they
    need at the measured 770 GB/s per direction (other ranks' pairs only)."""
    import torch
    T_r, Er = cfg.T // R, cfg.E // R
    H, I, E, k = cfg.H, cfg.I, cfg.E, cfg.k
    rs = moe.moe_shape(T_r, H, I, E, k, cfg.tile)
    ls = moe.moe_ep_local_shape(rs, R)
    rows = moe.moe_ep_pool_rows(rs, R)
    st = torch.cuda.current_stream().cuda_stream
    bf = torch.bfloat16
    own_arena = [torch.zeros(moe.moe_plan_arena_bytes(rs), dtype=torch.uint8, device=dev)
                 for _ in range(R)]
    own = [moe.moe_plan_bind(rs, a.data_ptr()) for a in own_arena]
    ep_arena = [torch.zeros(moe.moe_ep_arena_bytes(rs, R), dtype=torch.uint8, device=dev)
                for _ in range(R)]
    ep = [moe.moe_ep_bind(rs, R, a.data_ptr()) for a in ep_arena]
    pools = [torch.empty((rows, H), dtype=bf, device=dev) for _ in range(R)]
    acts = [torch.empty((rows, I), dtype=bf, device=dev) for _ in range(R)]
    ypools = [torch.empty((rows, H), dtype=bf, device=dev) for _ in range(R)]
    out = torch.empty((cfg.T, H), dtype=bf, device=dev)
    C = torch.zeros((R, E), dtype=torch.int32, device=dev)
    counts = [own_arena[r][own[r].counts - own_arena[r].data_ptr():][: 4 * E].view(torch.int32)
              for r in range(R)]
    xr = [x[r * T_r:(r + 1) * T_r] for r in range(R)]
    ir = [idx[r * T_r:(r + 1) * T_r] for r in range(R)]
    wr = [w[r * T_r:(r + 1) * T_r] for r in range(R)]
    # a rank's experts are a contiguous slice of the weights in either layout (the packed
    # tiles are expert-major)
    w1b = W1.numel() * W1.element_size() // E
    w2b = W2.numel() * W2.element_size() // E
    pp, yp = [p.data_ptr() for p in pools], [p.data_ptr() for p in ypools]
    # every stored row is counted on its owner's tile flag; the 'streaming' pass lets each
    # rank's GEMM A take tiles by their flags (here they are full: dispatches come first)
    flags = [e_.local.tile_flags for e_ in ep]
    fcfg = moe.moe_config(packed_weights=packed)

    def call(evs=None, fcfg=fcfg):
        def mark(i):
            if evs is not None:
                evs[i].record()
        mark(0)
        for r in range(R):
            moe.moe_plan(rs, ir[r].data_ptr(), own[r], 0, st)
        for r in range(R):
            C[r].copy_(counts[r])
        mark(1)
        for r in range(R):
            moe.moe_ep_layout(rs, R, r, C.data_ptr(), ep[r], pp[r], st)
        mark(2)
        for r in range(R):
            moe.moe_ep_dispatch(rs, R, r, xr[r].data_ptr(), own[r], ep[r], pp, st, flags)
        mark(3)
        for r in range(R):
            moe.moe_grouped_ffn(ls, pp[r], W1.data_ptr() + r * Er * w1b,
                                W2.data_ptr() + r * Er * w2b, ep[r].local, acts[r].data_ptr(),
                                yp[r], fcfg, st)
        mark(4)
        for r in range(R):
            moe.moe_ep_combine(rs, R, r, yp, wr[r].data_ptr(), own[r], ep[r],
                               out[r * T_r:(r + 1) * T_r].data_ptr(), st)
        mark(5)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    codes = [moe.moe_get_status(p)[0] for p in own] + \
        [moe.moe_get_status(e_.local)[0] for e_ in ep]
    if any(codes):
        raise RuntimeError(f"device status in the EP layer: {codes}")
    matches = bool(torch.equal(out.view(torch.int16), single_out.view(torch.int16)))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(reps)]
    for i in range(reps):
        call(evs[i])
    torch.cuda.synchronize()
    names = ("plan_and_exchange", "layout", "dispatch", "grouped_ffn", "combine")
    ph = {n: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(reps)) / reps
          for j, n in enumerate(names)}
    total = sum(evs[i][0].elapsed_time(evs[i][5]) for i in range(reps)) / reps
    # the same calls with streaming grouped FFNs (GEMM A waits on the tile flags; on this
    # one GPU they are full by then, and GEMM A leaves the dispatch SMs free)
    scfg = moe.moe_config(packed_weights=packed, streaming=1)
    out.zero_()
    call(None, scfg)
    torch.cuda.synchronize()
    s_matches = bool(torch.equal(out.view(torch.int16), single_out.view(torch.int16)))
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(reps)]
    for i in range(reps):
        call(sev[i], scfg)
    torch.cuda.synchronize()
    s_total = sum(sev[i][0].elapsed_time(sev[i][5]) for i in range(reps)) / reps
    codes = [moe.moe_get_status(p)[0] for p in own] + \
        [moe.moe_get_status(e_.local)[0] for e_ in ep]
    if any(codes):
        raise RuntimeError(f"device status in the streaming EP layer: {codes}")
    idx_h = idx.cpu().numpy()
    pairs = int((idx_h >= 0).sum())
    remote = []
    for r in range(R):
        e_ = idx_h[r * T_r:(r + 1) * T_r]
        e_ = e_[e_ >= 0]
        remote.append(int((e_ // Er != r).sum()))
    disp_b = cfg.T * H * 2 + pairs * H * 2
    comb_b = pairs * H * 2 + pairs * 8 + cfg.T * H * 2
    nv_b = max(remote) * H * 2
    res = {"ranks": R, "tokens_per_rank": T_r, "experts_per_rank": Er,
           "emulated": "all ranks on this GPU, their kernels one after another: peer "
                       "stores and loads are local HBM traffic; on R GPUs the ranks run side "
                       "by side and each rank's rows for other ranks cross NVLink",
           "ms_per_layer_call": total, "tokens_per_s": cfg.T / (total / 1e3),
           "phases_ms_per_call": {n: round(v, 5) for n, v in ph.items()},
           "dispatch_gbs": disp_b / (ph["dispatch"] / 1e3) / 1e9,
           "combine_gbs": comb_b / (ph["combine"] / 1e3) / 1e9,
           "dispatch_frac_hbm": disp_b / (ph["dispatch"] / 1e3) / 1e9 / peaks["hbm_gbs"],
           "combine_frac_hbm": comb_b / (ph["combine"] / 1e3) / 1e9 / peaks["hbm_gbs"],
           "matches_single_gpu_layer": matches,
           "streaming": {"ms_per_layer_call": s_total, "matches_single_gpu_layer": s_matches,
                         "note": "grouped FFNs with moe_config.streaming = 1 (tile flags)"},
           "nvlink": {"remote_pairs_per_rank_max": max(remote),
                      "bytes_per_rank_each_way_max": nv_b,
                      "dispatch_bound_ms_at_770_gbs": nv_b / 770e9 * 1e3,
                      "note": "on R GPUs each rank's dispatch stores, and its combine loads, "
                              "these bytes over NVLink (rows of pairs routed to other ranks)"},
           "gpu_launches_per_call": R * (3 + 1 + 5 + 1 + 2 + 1)}
    return res


def ensure_library(local: int) -> None:
    """Build the libraries when one is missing (a checkout without built libraries): the first
    local rank builds all three, the others wait until all three exist. Every build writes
    a file of its own and renames it into place, so a library that exists is complete."""
    if all(os.path.exists(p) for p in BUILT_LIBS):
        return
    if local == 0:
        import __graft_entry__
        __graft_entry__.build()
        return
    t0 = time.time()
    while time.time() - t0 < 900:
        if all(os.path.exists(p) for p in BUILT_LIBS):
            return
        time.sleep(1.0)
    raise RuntimeError("the libraries were not built in time by local rank 0")


def run_moe(args):
    import torch
    rank, world, local = dist_env()
    ensure_library(local)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    import combine_moe_plan_03_b200 as moe

    cfg = si.CONFIGS[args.workload]
    peaks, peak_src = load_peaks()
    streaming = 0 if args.streaming < 0 else args.streaming
    early = 0 if args.early_combine < 0 else args.early_combine
    mbs = cfg.micro_batches
    want_cpu = (world == 1 and rank == 0 and not args.no_cpu_baseline)

    # inputs: each rank takes its own tokens (micro-batch index offset by rank)
    xs, idxs, ws = [], [], []
    for m in range(mbs):
        g = rank * mbs + m
        xs.append(si.make_x(cfg, g))
        i_, w_ = si.make_routing(cfg, g)
        idxs.append(i_)
        ws.append(w_)
    if cfg.identity:
        W1 = W2 = None
        host = None
    else:
        W1, W2, host = upload_weights(cfg, dev, rank, world, keep_host=want_cpu)

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    dx = [dev_bf16(a) for a in xs]
    didx = [torch.from_numpy(a).to(dev) for a in idxs]
    dw = [torch.from_numpy(a).to(dev) for a in ws]
    buf = moe.MoELayerBuffers(cfg.T, cfg.H, max(cfg.I, 64), cfg.E, cfg.k, cfg.tile, device=dev,
                              identity=cfg.identity)
    packed = 1 if (args.packed and not cfg.identity) else 0
    ffn_kernel = args.ffn_kernel
    do_bwd = bool(args.backward) and not cfg.identity
    W1u, W2u = (W1, W2) if do_bwd else (None, None)   # the backward reads the given layout
    if packed:
        # one-time layout copy (as at model load), outside every timed region
        W1, W2 = buf.pack_weights(W1, W2)
        torch.cuda.empty_cache()
    calls = args.steps * mbs
    tev = moe.moe_timing_events_create(7 * calls)
    import ctypes
    ev_arrays = [(ctypes.c_void_p * 7)(*tev[7 * c: 7 * c + 7]) for c in range(calls)]
    early = early if not cfg.identity else 0
    cfgs = [moe.moe_config(streaming, 0, 0, packed, ffn_kernel,
                           ctypes.cast(ev_arrays[c], ctypes.c_void_p), None, early)
            for c in range(calls)]
    plain = moe.moe_config(streaming, 0, 0, packed, ffn_kernel, None, None, early)

    def step_plain():
        for m in range(mbs):
            buf.forward(dx[m], didx[m], dw[m], W1, W2, plain)

    for _ in range(args.warmup):
        step_plain()
    torch.cuda.synchronize()
    code, aux = moe.moe_get_status(buf.plan)
    if code != 0:
        raise RuntimeError(f"device status after warm-up: {moe.moe_strerror(code)} ({aux})")

    sampler = ClockSampler(physical_gpu_index(local))
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    sampler.mark(True)
    t_wall = time.perf_counter()
    c = 0
    for _ in range(args.steps):
        for m in range(mbs):
            buf.forward(dx[m], didx[m], dw[m], W1, W2, cfgs[c])
            c += 1
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    sampler.mark(False)
    barrier(world)
    clocks = sampler.stop()
    code, aux = moe.moe_get_status(buf.plan)
    if code != 0:
        raise RuntimeError(f"device status after timing: {moe.moe_strerror(code)} ({aux})")

    el = moe.moe_event_elapsed_ms
    total_ms = el(tev[0], tev[7 * (calls - 1) + 6])
    ph = {k: 0.0 for k in ("plan", "dispatch", "gemm_a", "gemm_y", "combine")}
    for c in range(calls):
        e = tev[7 * c: 7 * c + 7]
        ph["plan"] += el(e[0], e[1])
        ph["dispatch"] += el(e[1], e[2])
        ph["gemm_a"] += el(e[3], e[4])
        ph["gemm_y"] += el(e[4], e[5])
        ph["combine"] += el(e[5], e[6])
    ph = {k: v / calls for k, v in ph.items()}        # ms per launch (per layer call)
    red = reduce_max([total_ms] + [ph[k] for k in ph], dev, world)
    total_ms = red[0]
    ph = dict(zip(ph.keys(), red[1:]))

    tokens_step = cfg.T * mbs
    ms_step = total_ms / args.steps
    value = whole_job_tokens_per_s(world, tokens_step, ms_step)

    # ---------------- algorithmic work per layer call (averaged over the micro-batches)
    pairs = [int((i >= 0).sum()) for i in idxs]
    Ps = []
    for i in idxs:
        cnt = np.bincount(i[i >= 0].reshape(-1), minlength=cfg.E)
        Ps.append(int(((cnt + cfg.tile - 1) // cfg.tile * cfg.tile).sum()))
    # rows the grouped GEMMs compute: each expert's rows in ceil(c / 256) equal chunks (a
    # multiple of 16), every chunk's live rows rounded up to 16 (the MMA's N granularity)
    exec_rows = []
    for i in idxs:
        cnt = np.bincount(i[i >= 0].reshape(-1), minlength=cfg.E)
        rows = 0
        for c in cnt[cnt > 0].tolist():
            n = -(-c // 256)
            chunk = (-(-c // n) + 15) // 16 * 16
            rows += sum((min(chunk, c - r) + 15) // 16 * 16 for r in range(0, c, chunk))
        exec_rows.append(rows)
    exec_rows_m = float(np.mean(exec_rows))
    pairs_m = float(np.mean(pairs))
    n_live_experts = float(np.mean([len(np.unique(i[i >= 0])) for i in idxs]))
    P_m = float(np.mean(Ps))
    H, I, T = cfg.H, cfg.I, cfg.T
    disp_bytes = T * H * 2 + P_m * H * 2
    comb_bytes = pairs_m * H * 2 + T * H * 2 + pairs_m * 8
    dc_ms = ph["dispatch"] + ph["combine"]
    # with early combine the combine runs inside GEMM Y: no rate of its own
    dc_gbs = (disp_bytes + comb_bytes) / (dc_ms / 1000.0) / 1e9 if not early else None
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded SplitMix64/Box-Muller inputs, random-init expert weights)",
            "config": config_block(cfg, world),
            "weights": ("prepacked tiles (moe_pack_weights, once before timing)"
                        if packed else "as given: W1 [E,H,2I], W2 [E,I,H]"),
            "streaming": streaming, "ffn_kernel": ffn_kernel, "early_combine": early,
            "phases_ms_per_call": {k: round(v, 5) for k, v in ph.items()},
            "phases_mcycles_per_call": ({k: round(v * clocks["sm_mhz"] / 1000.0, 4)
                                         for k, v in ph.items()} if clocks.get("sm_mhz") else None),
            "dispatch_combine": {"bytes_per_call": disp_bytes + comb_bytes,
                                 "gbs": dc_gbs,
                                 "frac_hbm": dc_gbs / peaks["hbm_gbs"] if dc_gbs else None,
                                 "dispatch_gbs": disp_bytes / (ph["dispatch"] / 1e3) / 1e9,
                                 "combine_gbs": (comb_bytes / (ph["combine"] / 1e3) / 1e9
                                                 if not early else None),
                                 "padding_bytes": (P_m - pairs_m) * H * 2}}
    # the HBM ceilings of dispatch and combine on this GPU, from this library's own probe kernels
    probe = hbm_probe_rates(moe, dev)
    d_bound = copy_bound_ms(T * H * 2, P_m * H * 2, probe)
    c_bound = copy_bound_ms(pairs_m * H * 2 + pairs_m * 8, T * H * 2, probe)
    line["dispatch_combine"].update({
        "probe": probe,
        "dispatch_bound_ms": d_bound, "dispatch_frac_of_bound": d_bound / ph["dispatch"],
        "combine_bound_ms": c_bound,
        "combine_frac_of_bound": c_bound / ph["combine"] if not early else None,
        "bound_note": "shortest time at the probed write-only and copy rates (moe_hbm_probe)"})
    if not cfg.identity:
        flops_a = pairs_m * 4.0 * H * I
        flops_y = pairs_m * 2.0 * H * I
        ffn_ms = ph["gemm_a"] + ph["gemm_y"]
        ffn_tflops = (flops_a + flops_y) / (ffn_ms / 1e3) / 1e12
        exec_tflops = exec_rows_m * 6.0 * H * I / (ffn_ms / 1e3) / 1e12
        line["grouped_ffn"] = {"useful_tflops": ffn_tflops,
                               "frac_bf16_peak": ffn_tflops / peaks["bf16_tflops"],
                               "executed_tflops": exec_tflops,
                               "executed_frac_bf16_peak": exec_tflops / peaks["bf16_tflops"],
                               "weight_gbs": n_live_experts * 3 * H * I * 2 / (ffn_ms / 1e3)
                                             / 1e9,
                               "weight_frac_hbm": n_live_experts * 3 * H * I * 2
                                                  / (ffn_ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
        line["grouped_ffn"]["frac_bf16_sustained"] = ffn_tflops / peaks["bf16_tflops_sustained"]
        achieved = flops_a / (ph["gemm_a"] / 1e3) / 1e12
        # burst peak unless this run's clock record shows a seconds-long region held down by
        # the power cap (tensor_peak); both fractions beside it
        tpk, tsrc = tensor_peak(clocks, t_wall, peaks, peak_src)
        kname = ("ffn_gemm_pair_kernel<0>"
                 if (ffn_kernel or moe.MOE_FFN_DEFAULT) == moe.MOE_FFN_SM_PAIR
                 else "ffn_gemm_kernel<0>")
        # GEMM A does 2*rows flops per weight element (2 bytes): with fewer live rows per
        # expert than the ridge (sustained flop/s over HBM B/s) it streams weights from HBM.
        ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        rows_per_expert = pairs_m / max(n_live_experts, 1.0)
        if not streams_weights(pairs_m, n_live_experts, peaks):
            line["roofline"] = {"kernel": f"{kname} (GEMM A + SwiGLU)", "bound": "tensor",
                                "achieved": achieved, "peak": tpk, "unit": "TFLOP/s",
                                "frac": achieved / tpk,
                                "traffic": committed_traffic(kname, cfg.name),
                                "peak_source": tsrc,
                                "frac_of_burst": achieved / peaks["bf16_tflops"],
                                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                                "algorithmic": "useful flops pairs*4*H*I per launch"}
        else:
            a_bytes = (n_live_experts * H * 2 * I * 2 + pairs_m * H * 2 + pairs_m * I * 2)
            a_gbs = a_bytes / (ph["gemm_a"] / 1e3) / 1e9
            line["roofline"] = {"kernel": f"{kname} (GEMM A + SwiGLU)", "bound": "hbm",
                                "achieved": a_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": a_gbs / peaks["hbm_gbs"], "traffic": None,
                                "peak_source": f"{peak_src} HBM copy",
                                "algorithmic": "bytes per launch: W1 of the live experts "
                                               "+ live pool rows read + act rows written",
                                "rows_per_live_expert": rows_per_expert,
                                "ridge_flop_per_byte": ridge}
    else:
        achieved = disp_bytes / (ph["dispatch"] / 1e3) / 1e9
        line["roofline"] = {"kernel": "dispatch_kernel", "bound": "hbm", "achieved": achieved,
                            "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": achieved / peaks["hbm_gbs"],
                            "traffic": committed_traffic("dispatch_kernel", cfg.name),
                            "peak_source": f"{peak_src} HBM copy"}

    # ---------------- same-GPU A/B of the layer's options against the timed configuration
    if args.ab and not cfg.identity and world == 1:
        def variant(s_, e_):
            return moe.moe_config(s_, 0, 0, packed, ffn_kernel, None, None, e_)
        ab = ab_layer_ms(moe, buf, dx, didx, dw, W1, W2, {
            "timed": plain, "early_combine": variant(streaming, 1 - early),
            "streaming": variant(1 - streaming, early)})
        line["ab"] = {"ms_per_call": ab,
                      "note": "median of 4 alternating rounds of 10 calls; 'early_combine' and "
                              "'streaming' flip that one option of the timed configuration "
                              f"(early_combine={early}, streaming={streaming})"}

    # ---------------- router on the device (not part of the layer step: the layer takes
    # topk_idx / topk_w as inputs); timed on its own with the workload's logits
    if cfg.routing in ("softmax", "softmax_bias") and rank == 0:
        lg = si.normal_f32(cfg.seed, si.STREAM_LOGITS, 0, cfg.T * cfg.E).reshape(cfg.T, cfg.E)
        dl = torch.from_numpy(lg).to(dev)
        db = None
        if cfg.routing == "softmax_bias":
            db = torch.from_numpy(si.normal_f32(cfg.seed, si.STREAM_BIAS, 0, cfg.E,
                                                cfg.bias_sigma)).to(dev)
        ri = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
        rw = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
        rb = moe.MoELayerBuffers(cfg.T, 64, 64, cfg.E, cfg.k, cfg.tile, device=dev,
                                 identity=True)
        st = torch.cuda.current_stream().cuda_stream

        def rp():
            moe.moe_route_plan(rb.shape, dl.data_ptr(), db.data_ptr() if db is not None else 0,
                               ri.data_ptr(), rw.data_ptr(), rb.plan, 0, st)
        for _ in range(5):
            rp()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(50):
            rp()
        s1.record()
        torch.cuda.synchronize()
        rp_ms = s0.elapsed_time(s1) / 50
        line["router"] = {"route_plan_ms": rp_ms,
                          "kernels": 3 if 256 % cfg.k == 0 else 4,
                          "logits_gbs": cfg.T * cfg.E * 4 / (rp_ms / 1e3) / 1e9,
                          "matches_host_router": bool(np.array_equal(ri.cpu().numpy(), idxs[0])
                                                      if rank == 0 and mbs == 1 else True)}
        rb.close()

    # ---------------- backward of the layer (moe_backward), timed on its own after one forward:
    # every call recomputes the same gradients from the forward's plan, pool and ypool
    if do_bwd:
        line["backward"] = time_backward(moe, buf, cfg, dev, world, local, dx[0], didx[0], dw[0], W1,
                                         W2, W1u, W2u, packed, pairs[0], peaks, peak_src,
                                         args.steps)

    # ---------------- expert parallelism with R ranks emulated on this GPU (moe_ep_*)
    R = args.ep
    if (R > 1 and world == 1 and not cfg.identity and mbs == 1 and cfg.E % R == 0
            and cfg.T % R == 0):
        buf.forward(dx[0], didx[0], dw[0], W1, W2, plain)
        torch.cuda.synchronize()
        single = buf.out.clone()
        line["ep"] = time_ep(moe, cfg, dev, dx[0], didx[0], dw[0], W1, W2, packed, R, single,
                             peaks)
        del single
        torch.cuda.empty_cache()

    # ---------------- e2e: pinned host inputs in, result out, copies inside the timed region
    hx = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in xs]
    hidx = [torch.from_numpy(a).pin_memory() for a in idxs]
    hw = [torch.from_numpy(a).pin_memory() for a in ws]
    hout = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    # results go back on a copy stream from two device output buffers, so the copy of one
    # call's result overlaps the next call
    dout = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    done_ev = [torch.cuda.Event() for _ in range(2)]
    copied_ev = [torch.cuda.Event() for _ in range(2)]
    # two device copies of each input, so the copy of the next call's inputs (comm stream)
    # never overwrites what the current call's combine (compute stream) still reads
    bx = [torch.empty_like(dx[0]) for _ in range(2)]
    bi = [torch.empty_like(didx[0]) for _ in range(2)]
    bw = [torch.empty_like(dw[0]) for _ in range(2)]
    ncall = [0]

    def e2e_step():
        for m in range(mbs):
            j = ncall[0] & 1
            ncall[0] += 1
            with torch.cuda.stream(buf.comm):
                bx[j].copy_(hx[m], non_blocking=True)
                bi[j].copy_(hidx[m], non_blocking=True)
                bw[j].copy_(hw[m], non_blocking=True)
            buf.compute.wait_event(copied_ev[j])   # dout[j] was copied out two calls ago
            buf.forward(bx[j], bi[j], bw[j], W1, W2, plain, out=dout[j])
            done_ev[j].record(buf.compute)
            copy_stream.wait_event(done_ev[j])
            with torch.cuda.stream(copy_stream):
                hout[j].copy_(dout[j], non_blocking=True)
            copied_ev[j].record(copy_stream)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    s_ev = torch.cuda.Event(enable_timing=True)
    e_ev = torch.cuda.Event(enable_timing=True)
    s_ev.record(buf.comm)
    for _ in range(args.steps):
        e2e_step()
    buf.compute.wait_stream(copy_stream)
    e_ev.record(buf.compute)
    torch.cuda.synchronize()
    e2e_ms = reduce_max([s_ev.elapsed_time(e_ev)], dev, world)[0]
    h2d = mbs * (cfg.T * cfg.H * 2 + cfg.T * cfg.k * 8)
    d2h = mbs * cfg.T * cfg.H * 2
    line["e2e"] = {"value": world * tokens_step * args.steps / (e2e_ms / 1000.0),
                   "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    kernels_per_call = 5 if cfg.identity else (6 if early else 7)
    line["gpu_launches"] = kernels_per_call * calls   # the forward's timed region
    line["clocks"] = clocks
    if want_cpu and not cfg.identity:
        line["cpu_baseline"] = cpu_baseline(cfg, xs[0], idxs[0], ws[0], host,
                                            args.cpu_baseline_seconds)
    elif want_cpu:
        line["cpu_baseline"] = None
    moe.moe_events_destroy(tev)
    buf.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_moe(args)


if __name__ == "__main__":
    sys.exit(main())
