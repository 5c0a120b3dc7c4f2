#!/usr/bin/env python
"""Benchmark of the query-aware top-k block-sparse attention hot path on B200.

One step = the whole path over one batch of synthetic input: block pooling
and scoring, top-k selection (current block kept), and sparse attention over
the kept blocks, as consecutive library calls on one stream.  The headline
workload is the GQA prefill (B=1, 32 query / 8 KV heads, d=128, 32768
tokens, 64-token blocks, 16 history blocks + the current one).

Prints ONE JSON line (rank 0).  `value` is selected query-key pairs per
second over the whole step, aggregated over all ranks (each rank runs its own
independent problem: weak scaling, no collective on the data path).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

`--impl reference` times the CPU oracle (the plain definition of the method)
on the host cores, on a bounded sample of the same workload.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "selected QK-pairs/s (prefill step: pool+score+top-k+sparse attention)"
UNIT = "pairs/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 inputs run on the CUDA cores (fp32 FMA): 148 SMs x 128 fp32 lanes x 2 FLOP per FMA
# x 1.965 GHz (the maximum SM clock), in TFLOP/s
F32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="prefill_gqa_bf16")
    ap.add_argument("--cpu-rows", type=int, default=65536, help="query rows in the oracle CPU-baseline sample")
    ap.add_argument("--ref-rows", type=int, default=1024, help="query rows per reference-arm step")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-secondary", action="store_true", help="skip the other workloads' figures")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload batch (small profiling cases)")
    ap.add_argument("--variant", default="", choices=["", "pattern", "backward", "heads", "paged"],
                    help="a widened-path variant of the workload: prefill with the sink + local + top-k pattern, "
                         "the backward of the gated prefill, decode with one budget per head group, decode over "
                         "a paged cache")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# environment: ranks, peaks, clocks
# ----------------------------------------------------------------------------

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ----------------------------------------------------------------------------
# ranks: one process per GPU, each on its own independent problem (the path
# shards by (batch, KV group) with no exchange step); the process group only
# carries the barrier and the max-over-ranks timing.
# ----------------------------------------------------------------------------

def init_ranks(world: int, backend: str = "nccl", timeout_s: float = 120.0):
    """The process group for world > 1 (None otherwise); a short timeout so
    that ranks waiting for a rank that died end with an error."""
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def rank_workload(base, rank: int):
    """Rank r's independent problem: the same shapes, its own input seed."""
    return base.scaled(seed=base.seed + 1000 * rank, name=base.name) if rank else base


def reduce_over_ranks(dist, step_time: float, units: float, device=None):
    """(max step time over ranks, units summed over ranks); identity for one rank."""
    if dist is None:
        return step_time, units
    import torch
    t = torch.tensor([step_time], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def close_ranks(dist):
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clock, power and throttle reasons through NVML (read-only)
    every `period` seconds in a background thread."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index: int, period: float = 0.001):
        self.samples = []
        self.period = period
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self.max_mhz = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        power, n = None, 0
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                if n % 8 == 0:   # power changes slowly; read it on every eighth sample
                    power = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                n += 1
                self.samples.append((time.time(), mhz, reasons, power))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._ok:
            self.t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._ok:
            self.t.join(timeout=2)

    def summary(self, t0, t1):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win:   # region shorter than the sampling period: nearest samples
            win = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
        active = set()
        for _, _, r, _ in win:
            for name, const in self.REASONS.items():
                if r & getattr(self.nv, const):
                    active.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in win]) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(active),
                "power_w_max": max((s[3] for s in win if s[3] is not None), default=None),
                "samples": len(win)}


def wait_gpu(ev):
    """Wait for a recorded event by polling with short sleeps, so that the
    clock-sampling thread keeps the interpreter lock while the GPU works."""
    import torch
    while not ev.query():
        time.sleep(0.0005)
    torch.cuda.synchronize()


def capture_graph(fn):
    """A CUDA graph holding the launches of fn (the same C-ABI calls, captured
    once after warm-up).  Decode steps are replayed this way, as a serving
    loop issues them: the device-timed step then holds no host enqueue gaps."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        fn()
    torch.cuda.synchronize()
    return g


def profile_traffic(kernel_file: str, summary_name: str):
    """Per-launch DRAM traffic of the kernel from a committed ncu summary, or
    None when absent or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", summary_name)
    if not os.path.exists(path):
        return None, None
    text = open(path).read()
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    if not m_t or not m_h:
        return None, None
    return float(m_t.group(1)), m_h.group(1)


def prefill_kernel_of(w):
    """The prefill kernel the library runs for this shape: fp32 inputs run the
    SIMT kernel; bf16 units of an odd number of 128-row tiles (G*bs rows) go
    to the split-half kernel, even counts to the paired-tile kernel."""
    if w.dtype == "f32":
        return "attn_f32.cu", "attn_prefill_f32_kernel"
    tiles = (w.G * w.bs + 127) // 128
    if tiles % 2 == 1:
        return "attn_prefill_split.cu", "attn_prefill_kernel (split halves, one tile per item)"
    return "attn_prefill.cu", "attn_prefill_kernel (paired tiles)"


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "top_block_sparse_bsa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


# ----------------------------------------------------------------------------
# oracle sample (CPU baseline and reference arm)
# ----------------------------------------------------------------------------

def oracle_prefill_sample(w, q, k, v, group: int, rows: int, seed: int):
    """Times the oracle on one KV group: its selector (pool + score + top-k)
    over the group's whole sequence, and attention for `rows` random query
    rows of the group's heads.  Returns (pairs, seconds charged, detail)."""
    import oracle
    b, g = divmod(group, w.Hkv)
    G = w.G
    qs = q[b:b + 1, g * G:(g + 1) * G].float().cpu().numpy()
    ks = k[b:b + 1, g:g + 1].float().cpu().numpy()
    vs = v[b:b + 1, g:g + 1].float().cpu().numpy()
    t0 = time.perf_counter()
    _, _, s, idx, _ = oracle.prefill_select(qs, ks, 1, w.bs, w.kb)
    t_sel = time.perf_counter() - t0
    r = np.random.default_rng(seed)
    flat = r.choice(G * w.N, size=min(rows, G * w.N), replace=False).astype(np.int64)
    t1 = time.perf_counter()
    oracle.attend_prefill(qs, ks, vs, w.bs, idx, gate_scores=s if w.kind == "gated" else None, rows=flat)
    t_att = time.perf_counter() - t1
    # exact pairs of the sampled rows
    tpos = flat % w.N
    pairs = 0
    for t in tpos:
        i = int(t) // w.bs
        for j in idx[0, 0, i]:
            if j < 0:
                break
            pairs += w.bs if j < i else (int(t) % w.bs) + 1
    charged = t_att + t_sel * (len(flat) / (G * w.N))
    return pairs, charged, {"t_select_s": t_sel, "t_attend_s": t_att, "rows": int(len(flat))}


def prefill_config(w, world: int) -> dict:
    """The config object of a prefill line (both arms print the same one)."""
    in_mib = (w.B * w.Hq * w.N + 2 * w.B * w.Hkv * w.N) * w.d * (2 if w.dtype == "bf16" else 4) / 2**20
    l2_note = (f"inputs larger than L2 ({in_mib:.0f} MiB > 126 MiB)" if in_mib > 126 else
               f"inputs fit in L2 ({in_mib:.1f} MiB): L2-warm timing of a small workload")
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.N, "d": w.d,
            "block": w.bs, "budget": f"{w.kb}+current", "gated": w.kind == "gated",
            "global_batch": w.B * world, "parallelism": f"independent problems x{world}", "l2": l2_note,
            "dense_causal_pairs": w.N * (w.N + 1) // 2 * w.B * w.Hq}


def decode_config(w, world: int) -> dict:
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "ctx": w.N, "block": w.bs,
            "budget": w.kb, "global_batch": w.B * world, "parallelism": f"independent problems x{world}",
            "l2": "flushed before every step, outside the events: a 256 MiB write, then a 256 MiB read of "
                  "another buffer so that L2 holds clean unrelated lines",
            "launch": "CUDA graph replay of the C-ABI calls"}


def run_reference(args, world, rank):
    import bsa_workloads as W
    import oracle
    if rank != 0:
        return 0
    w = W.get(args.config)
    if w.kind in ("decode", "gist"):
        print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the oracle on the "
                          "prefill workloads only"}), flush=True)
        return 0
    inp = W.make_inputs(w, "cpu")
    threads = oracle.max_threads()
    pairs_total, secs_total = 0, 0.0
    for s in range(args.warmup + args.steps):
        group = s % (w.B * w.Hkv)
        pairs, secs, _ = oracle_prefill_sample(w, inp["q"], inp["k"], inp["v"], group, args.ref_rows, seed=s)
        if s >= args.warmup:
            pairs_total += pairs
            secs_total += secs
    value = pairs_total / secs_total
    sample = (f"per step: oracle selector (pool+score+top-k) on one KV group's full sequence, charged "
              f"pro rata, plus fp64 attention for {args.ref_rows} random query rows of that group")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": prefill_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def measure_prefill(w, dev, steps: int, warmup: int, peaks, peak_src, dist=None, pattern=None):
    """Times `steps` prefill steps (pool + score + top-k + sparse attention)
    of workload w on one stream, the attention launch of each step between
    its own pair of events.  Returns (figures, step object)."""
    import torch
    from top_block_sparse_bsa_b200 import accounting as acc
    from top_block_sparse_bsa_b200 import pipeline

    import bsa_workloads as W
    inp = W.make_inputs(w, dev)
    q, k, v = inp["q"], inp["k"], inp["v"]
    step = pipeline.PrefillStep(q, k, v, w.bs, w.kb, gated=(w.kind == "gated"), pattern=pattern)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        step.run(with_lse=False)
    torch.cuda.synchronize()
    idx = step.bufs["idx"].cpu().numpy()
    pairs = acc.prefill_pairs(idx, w.bs, w.G)
    flops = 4.0 * w.d * pairs
    kv_bytes = acc.prefill_kv_bytes(idx, w.bs, w.d, 2 if w.dtype == "bf16" else 4)
    full_pairs = acc.dense_pairs(w.N, causal=True) * w.B * w.Hq

    sampler = ClockSampler(dev.index or 0).start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ka = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    kb_ = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev0.record(stream)
    for s in range(steps):
        step.select()
        ka[s].record(stream)
        step.attend(with_lse=False)
        kb_[s].record(stream)
    ev1.record(stream)
    wait_gpu(ev1)
    t_wall1 = time.time()
    if dist:
        dist.barrier()
    sampler.stop()
    step_ms = ev0.elapsed_time(ev1) / steps
    attn_ms = statistics.mean(ka[s].elapsed_time(kb_[s]) for s in range(steps))

    sustained = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    burst = peaks["bf16_tflops"]
    achieved_tflops = flops / (attn_ms / 1e3) / 1e12
    hbm = peaks["hbm_gbs"]
    t_flop = flops / (burst * 1e12)
    t_hbm = kv_bytes / (hbm * 1e9)
    kfile, kname = prefill_kernel_of(w)
    traffic, sha = profile_traffic(kfile, f"{kfile[:-3]}_{w.name}.md")
    if sha is not None and sha != kernel_source_sha([kfile, "common.cuh", "tmem_wide.cuh"]):
        traffic = None
    # The burst peak is the denominator: the clock samples of the timed region
    # show the SM clock at its maximum with no power-cap reason, i.e. the
    # kernel does not run in the power-capped regime the sustained figure
    # describes.  The fraction of the sustained peak is reported alongside.
    if w.dtype == "f32":
        # the fp32 path is SIMT fp32 arithmetic, bounded by the CUDA cores' FMA rate
        t_flop = flops / (F32_FMA_PEAK_TFLOPS * 1e12)
        bound, peak, peak_note = "alu", F32_FMA_PEAK_TFLOPS, "derived: 148 SMs x 128 fp32 lanes x 2 x 1.965 GHz"
    else:
        bound, peak, peak_note = "tensor", burst, f"{peak_src} bf16 burst (cuBLAS GEMM timed alone)"
    roofline = {
        "bound": bound, "achieved": achieved_tflops, "peak": peak, "unit": "TFLOP/s",
        "frac": achieved_tflops / peak, "traffic": traffic,
        "peak_source": peak_note,
        "frac_of_sustained_peak": achieved_tflops / sustained if bound == "tensor" else None,
        "kernel": kname, "kernel_ms": attn_ms,
        "algorithmic_flop_per_launch": flops, "selected_kv_bytes_per_launch": kv_bytes,
        "roofline_time_ms": 1e3 * max(t_flop, t_hbm),
        "frac_of_roofline_time": (1e3 * max(t_flop, t_hbm)) / attn_ms,
        "hbm_gbs_on_selected_bytes": kv_bytes / (attn_ms / 1e3) / 1e9,
    }
    fig = {"step_ms": step_ms, "attn_ms": attn_ms, "pairs": pairs, "full_pairs": full_pairs,
           "roofline": roofline, "clocks": sampler.summary(t_wall0, t_wall1),
           "sparsity": acc.sparsity(pairs, full_pairs)}
    return fig, step


def run_prefill(args, world, rank, local, peaks, peak_src):
    import torch
    import bsa_workloads as W

    torch.cuda.set_device(local)
    dist = init_ranks(world)
    dev = torch.device("cuda", local)
    base = W.get(args.config)
    if args.batch:
        base = base.scaled(B=args.batch, name=base.name)
    w = rank_workload(base, rank)
    if args.variant == "backward":
        fig = measure_backward(w, dev, args.steps, args.warmup, peaks, peak_src)
        close_ranks(dist)
        if rank == 0:
            print(json.dumps(dict(fig, variant="backward", n_gpus=world, steps=args.steps, warmup=args.warmup,
                                  higher_is_better=False, data="synthetic")), flush=True)
        return 0
    pattern = None
    if args.variant == "pattern":
        w = w.scaled(kb=w.kb - 2, name=w.name)
        pattern = (1, 2)
    fig, step = measure_prefill(w, dev, args.steps, args.warmup, peaks, peak_src, dist, pattern=pattern)
    pairs = fig["pairs"]
    # whole job: the slowest rank's step, the pairs of every rank's problem
    step_ms, job_pairs = reduce_over_ranks(dist, fig["step_ms"], pairs, device=dev)
    value = job_pairs / (step_ms / 1e3)
    stream = torch.cuda.current_stream()
    q, k, v = step.q, step.k, step.v

    # end to end through the C ABI with host buffers: every step copies its
    # inputs from pinned host memory, runs the step and copies its output
    # back.  Two device buffer sets and three streams (copy in, compute, copy
    # out), as a serving loop would run it: step s's inputs go up while step
    # s-1 computes and step s-2's output comes down (the link is full
    # duplex); a set is refilled only after its previous output has left.
    e2e = None
    if args.e2e_steps > 0:
        from top_block_sparse_bsa_b200 import pipeline
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        ho = [torch.empty_like(hq).pin_memory() for _ in range(2)]
        other = pipeline.PrefillStep(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), w.bs, w.kb,
                                     gated=(w.kind == "gated"), pattern=pattern)
        sets = [step, other]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        n_it = args.e2e_steps + 2   # two untimed steps fill the pipeline
        for it in range(n_it):
            x = it % 2
            st = sets[x]
            if it == 2:
                e0.record(s_in)   # the timed region starts at step 2's copy-in, the pipeline running
            with torch.cuda.stream(s_in):
                if it >= 2:
                    s_in.wait_event(ev_out[x])
                st.q.copy_(hq, non_blocking=True)
                st.k.copy_(hk, non_blocking=True)
                st.v.copy_(hv, non_blocking=True)
                ev_in[x].record(s_in)
            stream.wait_event(ev_in[x])
            st.run(stream=stream, with_lse=False)
            ev_done[x].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[x])
                ho[x].copy_(st.bufs["o"], non_blocking=True)
                ev_out[x].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
        e2e_ms, _ = reduce_over_ranks(dist, e2e_ms, pairs, device=dev)
        h2d = (hq.numel() + hk.numel() + hv.numel()) * hq.element_size()
        e2e = {"value": job_pairs / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size(), "ms_per_step": e2e_ms,
               "pipelined": "two buffer sets; copy-in, compute and copy-out streams"}
        del hq, hk, hv, ho, other, sets

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        pairs_s, secs, detail = oracle_prefill_sample(w, q, k, v, group=0, rows=args.cpu_rows, seed=0)
        cpu_baseline = {"value": pairs_s / secs, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
                        "sample": (f"oracle selector (pool+score+top-k) on KV group 0's full {w.N}-token "
                                   f"sequence, charged pro rata, plus fp64 attention for {detail['rows']} "
                                   f"random query rows of that group"),
                        "detail": detail}
    del step, q, k, v
    torch.cuda.empty_cache()

    secondary = None
    if not args.no_secondary and world == 1:
        secondary = run_secondaries(dev, peaks, peak_src, exclude=w.name)

    close_ranks(dist)
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": prefill_config(w, world),
        "sparsity": fig["sparsity"],
        "roofline": fig["roofline"],
        "cpu_baseline": cpu_baseline,
        "e2e": e2e,
        "clocks": fig["clocks"],
        "gpu_launches": 4 * args.steps,   # pool (Q and K in one launch), score, top-k, attention
        "secondary": secondary,
    }
    print(json.dumps(line), flush=True)
    return 0


SECONDARY_STEPS, SECONDARY_WARMUP = 20, 5


def run_secondaries(dev, peaks, peak_src, exclude: str):
    """One figure set per other workload, each with its own roofline, step
    time and clock samples: the other prefill workloads (gated bf16, tiny
    fp32) through measure_prefill, decode and gist decode through
    measure_decode_like; then the widened path on the same shapes -- the
    prefill with a sink + local + top-k pattern, decode with one budget per
    head group, decode over a paged cache, the two-level gist decode, and the
    backward of the gated prefill."""
    import torch
    import bsa_workloads as W
    out = {}
    for name in ("gated_prefill_bf16", "tiny_prefill_f32", "decode_bf16", "gist_decode_bf16"):
        if name == exclude:
            continue
        w = W.get(name)
        if w.kind in ("decode", "gist"):
            out[name] = _decode_entry(w, dev, peaks, peak_src)
        else:
            out[name] = _prefill_entry(w, dev, peaks, peak_src)
        torch.cuda.empty_cache()
    c2 = W.get("prefill_gqa_bf16")
    out["prefill_gqa_bf16 pattern(sink 1, local 2, top 14)"] = _prefill_entry(c2.scaled(kb=14, name=c2.name), dev,
                                                                               peaks, peak_src, pattern=(1, 2))
    torch.cuda.empty_cache()
    dec = W.get("decode_bf16")
    out["decode_bf16 one budget per head group (96 x G)"] = _decode_entry(dec, dev, peaks, peak_src, "heads")
    torch.cuda.empty_cache()
    out["decode_bf16 paged (permuted pages)"] = _decode_entry(dec, dev, peaks, peak_src, "paged")
    torch.cuda.empty_cache()
    out["hssa_decode_bf16"] = _decode_entry(W.get("hssa_decode_bf16"), dev, peaks, peak_src)
    torch.cuda.empty_cache()
    out["gated_prefill_bf16 backward"] = measure_backward(W.get("gated_prefill_bf16"), dev, SECONDARY_STEPS,
                                                          SECONDARY_WARMUP, peaks, peak_src)
    torch.cuda.empty_cache()
    return out


def _decode_entry(w, dev, peaks, peak_src, variant: str = ""):
    fig = measure_decode_like(w, dev, SECONDARY_STEPS, SECONDARY_WARMUP, peaks, peak_src, variant=variant)
    return {"metric": "us per decode step", "us_per_step": fig["us"], "attn_us": fig["attn_us"],
            "roofline": fig["roofline"], "clocks": fig["clocks"], "config": decode_config(w, 1),
            "gpu_launches_per_step": fig["launches"]}


def _prefill_entry(w, dev, peaks, peak_src, pattern=None):
    fig, step = measure_prefill(w, dev, SECONDARY_STEPS, SECONDARY_WARMUP, peaks, peak_src, pattern=pattern)
    del step
    config = prefill_config(w, 1)
    if pattern is not None:
        config["pattern"] = {"sink": pattern[0], "local": pattern[1], "top": w.kb}
    return {"metric": METRIC, "value": fig["pairs"] / (fig["step_ms"] / 1e3), "unit": UNIT,
            "ms_per_step": fig["step_ms"], "roofline": fig["roofline"], "clocks": fig["clocks"],
            "config": config, "sparsity": fig["sparsity"], "gpu_launches_per_step": 4}


def measure_backward(w, dev, steps: int, warmup: int, peaks, peak_src):
    """The backward of the gated prefill on workload w: one forward (with its
    LSE) on the selected blocks, then `steps` timed backward calls.  FLOPs per
    call: 10 d per causal pair (Q K^T, dO V^T, dV, dQ, dK; the recomputation
    of Q K^T and dO V^T in the second pass and the query-major pass's extra
    sweep that forms D are not counted); the products run on the bf16 tensor
    cores, so the bound is the measured bf16 GEMM rate (burst: the call is
    timed alone)."""
    import torch
    import bsa_workloads as W
    from top_block_sparse_bsa_b200 import accounting as acc
    from top_block_sparse_bsa_b200 import pipeline
    inp = W.make_inputs(w, dev)
    step = pipeline.PrefillStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb, gated=(w.kind == "gated"))
    step.run()
    g = torch.Generator(device=dev).manual_seed(3)
    d_o = torch.randn(inp["q"].shape, generator=g, device=dev).to(torch.bfloat16)
    for _ in range(warmup):
        step.backward(d_o)
    torch.cuda.synchronize()
    pairs = acc.prefill_pairs(step.bufs["idx"].cpu().numpy(), w.bs, w.G)
    flops = 10.0 * w.d * pairs
    sampler = ClockSampler(dev.index or 0).start()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        step.backward(d_o)
    e1.record(stream)
    wait_gpu(e1)
    t1 = time.time()
    sampler.stop()
    ms = e0.elapsed_time(e1) / steps
    achieved = flops / (ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    del step, inp, d_o
    return {"metric": "ms per backward call", "ms_per_call": ms, "config": prefill_config(w, 1),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "peak_source": peak_src,
                         "algorithmic_flop_per_call": flops,
                         "kernel": "bsa_gated_attn_bwd (5 launches: gate, transpose, dq_tc, dkv_tc, dsel)"},
            "clocks": sampler.summary(t0, t1), "gpu_launches_per_step": 5}


def measure_decode_like(w, dev, steps: int, warmup: int, peaks, peak_src, dist=None, variant: str = ""):
    """Decode or gist-decode workload: microseconds per step and HBM GB/s
    over the bytes the attention must read, L2 flushed before every step."""
    import torch
    from top_block_sparse_bsa_b200 import accounting as acc
    from top_block_sparse_bsa_b200 import pipeline
    import bsa_workloads as W
    inp = W.make_inputs(w, dev)
    if w.kind == "decode" and variant == "heads":
        step = pipeline.HeadBudgetDecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb * w.G)
        step.pool_cache()
        select = step.select
        attend = lambda: step.attend(with_lse=False)   # noqa: E731
        launches = 5   # per-head scores, joint top-k | union lists, split-K attention, combine
        attn_kernel = "gist_union_kernel (no gists) + attn_decode_kernel + combine_kernel"
    elif w.kind == "decode" and variant == "paged":
        ref = pipeline.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
        ref.pool_cache()
        nb = w.N // w.bs
        perm = torch.from_numpy(np.random.default_rng(7).permutation(w.B * nb).astype(np.int32)).to(dev)
        table = perm.view(w.B, nb)
        pools = []
        for name in ("k", "v"):
            blocks = inp[name].view(w.B, w.Hkv, nb, w.bs, w.d).permute(0, 2, 1, 3, 4).reshape(w.B * nb, w.Hkv,
                                                                                                w.bs, w.d)
            pool = torch.empty_like(blocks)
            pool[perm.long()] = blocks
            pools.append(pool)
            del blocks
        kbar = ref.bufs["kbar"]
        del ref
        inp = {"q": inp["q"]}
        torch.cuda.empty_cache()
        step = pipeline.PagedDecodeStep(inp["q"], pools[0], pools[1], table, w.bs, w.kb)
        step.bufs["kbar"].copy_(kbar)
        del kbar
        select = step.select
        attend = lambda: step.attend(with_lse=False)   # noqa: E731
        launches = 3   # fused select | split-K attention over the block table, combine
        attn_kernel = "attn_decode_kernel (paged) + combine_kernel"
    elif w.kind == "decode":
        step = pipeline.DecodeStep(inp["q"], inp["k"], inp["v"], w.bs, w.kb)
        step.pool_cache()
        select = step.select
        attend = lambda: step.attend(with_lse=False)   # noqa: E731
        launches = 3   # fused score + top-k | split-K attention, combine
        attn_kernel = "attn_decode_kernel (+ combine_kernel)"
    elif w.kind == "hssa":
        step = pipeline.HssaStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], inp["mk"], inp["mv"], w.bs,
                                 W.HSSA_GROUPS_KEPT, w.kb)
        select = lambda: step.run(with_lse=False)   # noqa: E731  (the whole step in one call)
        attend = None
        launches = 6   # meta scores, top-km, group gist scores + top-k, union, attention, combine
        attn_kernel = "whole two-level gist step (one call)"
    else:
        step = pipeline.GistStep(inp["q"], inp["k"], inp["v"], inp["gk"], inp["gv"], w.bs, w.kb)
        select = lambda: step.run(with_lse=False)   # noqa: E731  (the whole step in one call)
        attend = lambda: step.run(idx_in=step.bufs["idx"], with_lse=False)   # noqa: E731
        launches = 4   # gist score, top-k, split-K attention (union built inside), combine
        attn_kernel = "attn_decode_kernel (the group's union built in the kernel) + combine_kernel"
    # L2 flush between steps: a 256 MiB write evicts every input line, and a
    # 256 MiB read of a second buffer then evicts the write's dirty lines, so
    # the timed step neither finds its inputs in L2 nor pays for writing back
    # the flush (measured: a write-only flush adds 11 us to the decode step and
    # 13 us to the gist step, the write-back of about 120 MB of dirty lines).
    flush_w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(256 * 1024 * 1024 // 8, dtype=torch.int64, device=dev)

    def flush(s):
        flush_w.fill_(s & 0xFF)
        flush_r.sum()
    for _ in range(warmup):
        select()
        if attend is not None:
            attend()
    torch.cuda.synchronize()
    idx = step.bufs["idx"].cpu().numpy()
    if w.kind == "decode" and variant == "heads":
        nbytes = acc.heads_kv_bytes(idx, w.G, w.bs, w.d, 2)
    elif w.kind == "decode":
        nbytes = acc.decode_kv_bytes(idx, w.bs, w.d, 2)
    elif w.kind == "hssa":
        nbytes = acc.hssa_kv_bytes(idx, step.bufs["meta_idx"].cpu().numpy(), w.G, w.bs, w.d, 2)
    else:
        nbytes = acc.gist_kv_bytes(idx, w.G, w.bs, w.N // w.bs, w.d, 2)
    # Each step is replayed from CUDA graphs of the C-ABI calls, L2 flushed
    # first.  The timed step is one graph holding the whole step.  The
    # attention part is timed in a second pass: decode replays the selection
    # graph and then the attention graph, timing the latter (its launch is
    # queued behind the selection, as inside a step); gist (whose step is one
    # call) replays the attention-only call (its own indices injected) after
    # another L2 flush, queued behind that flush.
    if w.kind == "decode":
        g_step = capture_graph(lambda: (select(), attend()))
    else:
        g_step = capture_graph(select)
    g_sel = capture_graph(select) if w.kind == "decode" else None
    g_att = capture_graph(attend) if attend is not None else g_step
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    sampler = ClockSampler(dev.index or 0).start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for s in range(steps):
        flush(s)
        ev[s][0].record(stream)
        g_step.replay()
        ev[s][1].record(stream)
    wait_gpu(ev[-1][1])
    t1 = time.time()
    sampler.stop()
    us = statistics.mean(1e3 * e[0].elapsed_time(e[1]) for e in ev)
    ea = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for s in range(steps):
        flush(s)
        if g_sel is not None:
            g_sel.replay()
        ea[s][0].record(stream)
        g_att.replay()
        ea[s][1].record(stream)
    wait_gpu(ea[-1][1])
    attn_us = statistics.mean(1e3 * e[0].elapsed_time(e[1]) for e in ea)
    del g_step, g_sel, g_att
    gbs = nbytes / (attn_us / 1e6) / 1e9
    traffic, sha = profile_traffic("attn_decode.cu", f"attn_decode_{w.name}.md")
    if sha is not None and sha != kernel_source_sha(["attn_decode.cu", "common.cuh"]):
        traffic = None
    if variant or w.kind == "hssa":
        traffic = None   # no committed counter summary for these variants
    roofline = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                "kernel": attn_kernel, "kernel_us": attn_us, "selected_kv_bytes_per_launch": nbytes,
                "step_gbs": nbytes / (us / 1e6) / 1e9, "roofline_us": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e6}
    fig = {"us": us, "attn_us": attn_us, "nbytes": nbytes, "roofline": roofline,
           "clocks": sampler.summary(t0, t1), "launches": launches}
    del step, inp, flush_w, flush_r
    return fig


def run_decode_like(args, world, rank, local, peaks, peak_src):
    import torch
    import bsa_workloads as W
    torch.cuda.set_device(local)
    dist = init_ranks(world)
    dev = torch.device("cuda", local)
    base = W.get(args.config)
    if args.batch:
        base = base.scaled(B=args.batch, name=base.name)
    w = rank_workload(base, rank)
    fig = measure_decode_like(w, dev, args.steps, args.warmup, peaks, peak_src, dist, variant=args.variant)
    # whole job: every rank runs its own batch; a step takes the slowest rank's time
    us, _ = reduce_over_ranks(dist, fig["us"], 1.0, device=dev)
    attn_us, _ = reduce_over_ranks(dist, fig["attn_us"], 1.0, device=dev)
    close_ranks(dist)
    if rank != 0:
        return 0
    roofline = dict(fig["roofline"])
    gbs = fig["nbytes"] / (attn_us / 1e6) / 1e9
    roofline.update(achieved=gbs, frac=gbs / peaks["hbm_gbs"], kernel_us=attn_us,
                    step_gbs=fig["nbytes"] / (us / 1e6) / 1e9)
    line = {
        "metric": "us per decode step", "value": us, "unit": "us", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": decode_config(w, world),
        "roofline": roofline,
        "clocks": fig["clocks"], "gpu_launches": fig["launches"] * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    peaks, src = load_peaks()
    import bsa_workloads as W
    if W.get(args.config).kind in ("decode", "gist", "hssa"):
        return run_decode_like(args, world, rank, local, peaks, src)
    return run_prefill(args, world, rank, local, peaks, src)


if __name__ == "__main__":
    sys.exit(main())
