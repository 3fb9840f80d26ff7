#!/usr/bin/env python
"""Benchmark of one SparseSAM encoder block's hot path on B200.

A step is one pass of the whole path -- Sobel score, stripe-sort permutation, Stripe-Sort sparse
attention, Residual-Consistency MLP -- over one batch of the named synthetic workload (default:
SAM ViT-H global block, 4 x 64x64 tokens, 16 heads x 80, density 0.3, MLP 1280->5120->1280, the
largest single-block configuration). The SAM ViT-B global and windowed blocks are measured the same
way and reported under "also".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One process per GPU (torchrun for N > 1). The path has no exchange step: each rank runs an
independent replica of the workload (weak scaling) and the job's throughput is all ranks' tokens
over the slowest rank's device time. Rank 0 prints one JSON line.

`value` times the steps with inputs resident on the device (rotating over input sets larger than
L2). `e2e` times the same steps through the same calls with every step's inputs copied in from
pinned host memory and its results (out, x) read back, pipelined the way a serving loop runs:
the copy-in of one step, the compute of the previous one and the read-back of the one before
overlap on three streams over two device buffer sets.

--impl reference times the float64 CPU oracle (the only reference this method has) on the host
cores, on a bounded sample of the same workload, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from structured_activation_sparsity_b200 import workloads  # noqa: E402

METRIC = "Stripe-Sort attn + RC-MLP tokens/s per block; effective TFLOP/s vs bf16 peak"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024

# dram__bytes_read.sum + dram__bytes_write.sum of one attention launch per workload, from an ncu
# capture of the current attention kernel on that workload (profiles/ names the capture). A
# workload is absent (traffic null) until its capture is taken again after a kernel change.
ATTN_TRAFFIC_BYTES = {
    "vith_global": 125_934_848 + 21_374_464,    # k_attn_pair<80>: profiles/attn_pair_vith_global.md
    "vitb_global": 18_952_960 + 0,              # k_attn_pair<64>: profiles/attn_pair_vitb_global.md
    "vitb_window": 90_458_880 + 9_328_384,      # k_attn_pairs: profiles/attn_pairs_vitb_window.md
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d["bf16_tflops_sustained"], d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ------------------------------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.period, self.ok = [], period_s, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(device_index)
            h = None
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                dom = getattr(props, "pci_domain_id", 0)
                dev = getattr(props, "pci_device_id", 0)
                try:
                    h = pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08X}:{bus:02X}:{dev:02X}.0")
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report what we could not sample
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
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

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0, "note": getattr(self, "err", "no samples")}
        mhz = [m for m, _ in self.samples]
        seen = 0
        for _, r in self.samples:
            seen |= r
        reasons = [k for k, bit in self.REASONS.items() if seen & bit and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ------------------------------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline leg)
# ------------------------------------------------------------------------------------------------
def cpu_sample(wl, min_seconds: float = 10.0):
    """Time the float64 oracle on a bounded sample of the workload; return per-step seconds for
    the full workload and a description. The sample: image 0's score, permutation and keep list;
    attention of unit 0 for `hs` heads; the RC-MLP of image 0's kept rows. Per-step time is scaled
    linearly to all units, heads and images."""
    from oracle import sparsesam_oracle as O
    from structured_activation_sparsity_b200 import synth

    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    lum = synth.luminance(wl)[:1]
    g = np.random.default_rng(wl.seed)
    hs = min(wl.heads, 2)
    shape = (1, wl.unit_tokens, hs, wl.head_dim)
    q, k, v = (synth.bf16_to_f64(synth.to_bf16(g.standard_normal(shape, dtype=np.float32)))
               for _ in range(3))
    x, w1, b1, w2, b2 = synth.mlp_params(wl.with_(batch=1))
    x, w1, w2 = (synth.bf16_to_f64(synth.to_bf16(a)) for a in (x, w1, w2))
    geo = O.Geometry(1, wl.grid_h, wl.grid_w, wl.mode, wl.window)
    reps, t_sp, t_at, t_mlp = 0, 0.0, 0.0, 0.0
    t_begin = time.perf_counter()
    while reps == 0 or time.perf_counter() - t_begin < min_seconds:
        t0 = time.perf_counter()
        score = O.sobel_score(lum)
        perm, _ = O.stripe_sort(score, geo)
        keep = O.keep_list(score, wl.density)
        t1 = time.perf_counter()
        O.attention(q, k, v, perm[:1], wl.density)
        t2 = time.perf_counter()
        O.rcmlp(x, w1, None, w2, None, keep)
        t3 = time.perf_counter()
        t_sp, t_at, t_mlp, reps = t_sp + t1 - t0, t_at + t2 - t1, t_mlp + t3 - t2, reps + 1
    t_sp, t_at, t_mlp = t_sp / reps, t_at / reps, t_mlp / reps
    step = (t_sp * wl.batch + t_at * wl.units * wl.heads / hs + t_mlp * wl.batch)
    desc = (f"oracle on image 0 (score+perm+keep), unit 0 x {hs}/{wl.heads} heads (attention), "
            f"image 0's {O.keep_count(wl.density, wl.tokens_per_image)} kept rows (MLP); "
            f"{reps} reps, scaled linearly to {wl.batch} image(s), {wl.units} unit(s), "
            f"{wl.heads} heads")
    return step, desc, cores, reps * (t_sp + t_at + t_mlp)


def run_reference(args, wl, rank):
    if rank != 0:
        return
    steps_t = []
    desc = cores = None
    for _ in range(args.warmup if args.warmup < 1 else 1):
        cpu_sample(wl, min_seconds=0.0)
    for _ in range(args.steps):
        step, desc, cores, _ = cpu_sample(wl, min_seconds=0.0)
        steps_t.append(step)
    per_step = sum(steps_t) / len(steps_t)
    value = wl.batch * wl.tokens_per_image / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl, args, extra=None):
    c = {"workload": wl.name, "batch": wl.batch, "grid": f"{wl.grid_h}x{wl.grid_w}",
         "mode": wl.mode, "heads": wl.heads, "head_dim": wl.head_dim, "density": wl.density,
         "mlp": f"{wl.dim}->{wl.hidden}->{wl.dim}", "parallelism": f"replicas x{args.gpus}"}
    if wl.mode == "window":
        c["window"] = wl.window
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------
def make_sets(wl, n_sets, dev, density=None):
    import torch
    from structured_activation_sparsity_b200 import synth
    from structured_activation_sparsity_b200.hotpath import HotPath

    lum = torch.from_numpy(synth.luminance(wl))
    q, k, v = (synth.to_bf16(a) for a in synth.qkv(wl))
    mlp = [synth.to_bf16(a) for a in synth.mlp_params(wl)]
    sets = []
    for _ in range(n_sets):
        hp = HotPath(wl, device=dev, density=density)
        hp.load(lum, q, k, v, *mlp)
        sets.append(hp)
    return sets, (lum, q, k, v, mlp)


def kernel_bytes(wl, pat):
    """Algorithmic DRAM bytes per launch of the bandwidth-bound kernels of one step."""
    T = wl.batch * wl.grid_h * wl.grid_w              # real tokens
    units_tokens = wl.units * wl.unit_tokens          # tokens incl. window pads
    K = wl.batch * pat.keep
    row = wl.heads * wl.head_dim * 2                  # one token's bf16 Q (or K, V) row
    return {
        # lum in, score out, perm and inv out, keep out
        "score_rank": T * 4 + T * 8 + units_tokens * 8 + K * 4,
        "sobel_score": T * 4 + T * 8,
        "stripe_rank": T * 8 + units_tokens * 8 + K * 4,
        "gather_qkv": 2 * 3 * units_tokens * row,     # Q, K, V read once and written once
        "unpermute_out": 2 * units_tokens * row,      # the permuted output read, out written
        "gather_rows": 2 * K * wl.dim * 2,            # kept rows of x read and written
    }


def set_bytes(hp):
    ts = [hp.lum, hp.score, hp.perm, hp.inv, hp.keep, hp.q, hp.k, hp.v, hp.out, hp.x, hp.w1,
          hp.w2, hp.ws_block]
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


def time_steps(sets, steps, stream, dist=None):
    import torch
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(steps):
        sets[i % len(sets)].step(stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return ev0.elapsed_time(ev1) / 1e3


def max_over_ranks(x, dist, dev):
    """The slowest rank's time: the job is done when every replica is."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_step: int, steps: int, seconds: float) -> float:
    """Weak scaling: every rank runs its own replica, so the job processes world x the units."""
    return world * units_per_step * steps / seconds


def time_attn_kernel(sets, launches, stream, warmup=3):
    """Average duration of the attention kernel alone: CUDA events on the launching stream around
    `launches` back-to-back launches over the rotating input sets (their workspaces hold the
    permuted Q, K, V their last step left), so that consecutive launches overlap as inside a step
    (programmatic dependent launch) and no per-launch event stands between them."""
    import torch
    for i in range(warmup):
        sets[i % len(sets)].attn_kernel_step(stream)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(launches):
        sets[i % len(sets)].attn_kernel_step(stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1) * 1e3 / launches


def measure(args, wl, dist, dev, stream, world):
    """The timed steps of one workload and the per-kernel figures behind them."""
    import torch
    from structured_activation_sparsity_b200 import _lib as L

    bf16_peak, _, hbm_peak, peak_src = peaks()
    probe, _ = make_sets(wl, 1, dev)
    per_set = set_bytes(probe[0])
    n_sets = max(2, math.ceil(3 * L2_BYTES / per_set))
    sets = probe + make_sets(wl, n_sets - 1, dev)[0]
    pat = sets[0].pattern
    tokens_per_step = wl.batch * wl.tokens_per_image
    attn_flops = workloads.attn_flops(wl.units, wl.unit_tokens, wl.heads, wl.head_dim, pat.rho)
    mlp_flops = workloads.mlp_flops(wl.batch * pat.keep, wl.dim, wl.hidden)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            sets[i % n_sets].step(stream)
    torch.cuda.synchronize()
    if L.sparsesam_device_status(stream) != L.SS_OK:
        raise RuntimeError("a device wait timed out during warm-up")

    # ---- timed region: exactly K steps --------------------------------------------------------
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    n0 = L.sparsesam_launch_count()
    t = time_steps(sets, args.steps, stream, dist)
    launches = L.sparsesam_launch_count() - n0
    clocks.stop()
    t = max_over_ranks(t, dist, dev)
    ms_per_step = t / args.steps * 1e3
    value = job_throughput(world, tokens_per_step, args.steps, t)

    # ---- per-kernel durations: the same K steps again with an event pair around every launch ----
    # (the events keep each launch from overlapping its neighbours, so these include launch
    # latency; the attention's own figure below has no event between launches)
    L.sparsesam_trace_start(8 * args.steps + 16)
    time_steps(sets, args.steps, stream, dist)
    recs = L.sparsesam_trace_stop()
    per_kernel = {}
    for name, ms in recs:
        per_kernel.setdefault(name, []).append(ms)
    kernels = {n: {"launches": len(v), "avg_us_traced": 1e3 * sum(v) / len(v)}
               for n, v in per_kernel.items()}
    moved = kernel_bytes(wl, pat)
    for n, nbytes in moved.items():
        if n in kernels:
            gbs = nbytes / (kernels[n]["avg_us_traced"] * 1e-6) / 1e9
            kernels[n].update({"bytes": nbytes, "gbs_traced": gbs, "frac_hbm_traced": gbs / hbm_peak})

    # ---- the attention kernel (the roofline's kernel): its CUDA-event duration in the traced
    # steps (events on the launching stream around each launch, so the figure includes the
    # launch's own start-up); also the attention call without its gather, back to back ------------
    # (a shape whose last round of pairs is split into pieces also runs merge_pieces, which
    # finishes those pairs: it counts toward the attention's time)
    attn_us = kernels["attn"]["avg_us_traced"]
    if "merge_pieces" in kernels:
        attn_us += kernels["merge_pieces"]["avg_us_traced"]
    loop_us = time_attn_kernel(sets, max(50, args.steps), stream)
    kernels["attn"]["avg_us_back_to_back_with_unpermute"] = loop_us
    achieved = attn_flops / (attn_us * 1e-6) / 1e12
    roofline = {"bound": "tensor", "kernel": "attn", "achieved": achieved, "peak": bf16_peak,
                "unit": "TFLOP/s", "frac": achieved / bf16_peak,
                "traffic": ATTN_TRAFFIC_BYTES.get(wl.name),
                "peak_source": f"{peak_src} bf16 burst",
                "algorithmic_flops_per_launch": attn_flops,
                "timing": "CUDA events on the launching stream around each attention launch "
                          "(plus merge_pieces where the shape splits pairs) of "
                          f"the {args.steps} traced steps"}
    if L.sparsesam_device_status(stream) != L.SS_OK:
        raise RuntimeError("a device wait timed out during timing")
    return {"sets": sets, "n_sets": n_sets, "per_set": per_set, "pat": pat, "value": value,
            "t": t, "ms_per_step": ms_per_step, "launches": launches, "clocks": clocks,
            "kernels": kernels, "roofline": roofline, "attn_flops": attn_flops,
            "mlp_flops": mlp_flops, "tokens_per_step": tokens_per_step}


def run_ours(args, wl, rank, world, local_rank, dist):
    import torch
    from structured_activation_sparsity_b200 import _lib as L

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    m = measure(args, wl, dist, dev, stream, world)
    sets, n_sets, pat = m["sets"], m["n_sets"], m["pat"]
    t, value, tokens_per_step = m["t"], m["value"], m["tokens_per_step"]

    # ---- dense comparison: the same kernels at density 1.0 -----------------------------------------
    dense_sets = make_sets(wl, n_sets, dev, density=1.0)[0]
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            dense_sets[i % n_sets].step(stream)
    td = max_over_ranks(time_steps(dense_sets, args.steps, stream, dist), dist, dev)
    dense_value = job_throughput(world, tokens_per_step, args.steps, td)
    dpat = dense_sets[0].pattern
    dense_flops = (workloads.attn_flops(wl.units, wl.unit_tokens, wl.heads, wl.head_dim, dpat.rho)
                   + workloads.mlp_flops(wl.batch * dpat.keep, wl.dim, wl.hidden))
    del dense_sets

    # ---- end to end: pinned host inputs in, results out, through the same C-ABI calls ------------
    # Pipelined over two device buffer sets and three streams, as a serving loop runs: step i's
    # inputs are copied in (one stream) while step i-1 computes (the compute stream) and step
    # i-2's results are read back (a third stream). Every step copies all of its inputs in and all
    # of its results (out, x) back.
    e2e_sets = sets[:2]
    host_in = [t_.detach().to("cpu").pin_memory() for t_ in e2e_sets[0].input_tensors()]
    host_out = [[torch.empty(h.out.shape, dtype=h.out.dtype).pin_memory(),
                 torch.empty(h.x.shape, dtype=h.x.dtype).pin_memory()] for h in e2e_sets]
    h2d = sum(x.numel() * x.element_size() for x in host_in)
    d2h = sum(x.numel() * x.element_size() for x in host_out[0])
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in e2e_sets]
    ev_c = [torch.cuda.Event() for _ in e2e_sets]
    ev_out = [torch.cuda.Event() for _ in e2e_sets]

    def e2e_step(i):
        b = i % len(e2e_sets)
        h = e2e_sets[b]
        s_in.wait_event(ev_out[b])   # set b's previous results have been read back
        with torch.cuda.stream(s_in):
            for dst, src in zip(h.input_tensors(), host_in):
                dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        h.step(stream)
        ev_c[b].record(stream)
        s_out.wait_event(ev_c[b])
        with torch.cuda.stream(s_out):
            host_out[b][0].copy_(h.out, non_blocking=True)
            host_out[b][1].copy_(h.x, non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(max(3, args.warmup // 4)):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    ev1.record(s_out)   # after the last read-back, which follows every other step's work
    torch.cuda.synchronize()
    te = max_over_ranks(ev0.elapsed_time(ev1) / 1e3, dist, dev)
    e2e_value = job_throughput(world, tokens_per_step, args.steps, te)
    if L.sparsesam_device_status(stream) != L.SS_OK:
        raise RuntimeError("a device wait timed out during timing")
    del sets, e2e_sets, m["sets"]
    torch.cuda.empty_cache()

    # ---- the other single-block workloads, measured the same way (extra keys of the line) -------
    also = {}
    for name in [n for n in args.also.split(",") if n and n != wl.name]:
        w2 = workloads.get(name)
        m2 = measure(args, w2, dist, dev, stream, world)
        also[name] = {"value": m2["value"], "unit": UNIT, "ms_per_step": m2["ms_per_step"],
                      "config": config_of(w2, args, {"realised_density": m2["pat"].rho}),
                      "roofline": m2["roofline"], "clocks": m2["clocks"].summary(),
                      "gpu_launches": int(m2["launches"]),
                      "effective_tflops": (m2["attn_flops"] + m2["mlp_flops"]) * args.steps
                      * world / m2["t"] / 1e12}
        del m2
        torch.cuda.empty_cache()

    # ---- the variants (attention only), measured the same way (extra key) --------------------
    variants = None if args.no_stack else measure_variants(args, dev, stream,
                                                           max(10, min(args.steps, 50)),
                                                           args.warmup)

    # ---- the ViT-L encoder stack of full blocks at the density sweep (extra key) --------------
    stack = None
    if not args.no_stack:
        stack = {"model": "vitl_24_blocks", "batch": VITL_STACK["batch"],
                 "sweep": measure_stack(args, dev, stream, (1.0, 0.5, 0.4, 0.3),
                                        max(5, min(args.steps, 20)), args.warmup)}

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(wl, args, {
            "l2": f"{n_sets} rotating input sets of {m['per_set'] / 2**20:.0f} MiB (> 3x L2)",
            "realised_density": pat.rho, "mlp_tokens_per_image": pat.keep}),
        "clocks": m["clocks"].summary(),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": int(m["launches"]),
        "effective_tflops": (m["attn_flops"] + m["mlp_flops"]) * args.steps * world / t / 1e12,
        "roofline": m["roofline"],
        "kernels": m["kernels"],
        "dense": {"value": dense_value, "unit": UNIT, "ms_per_step": td / args.steps * 1e3,
                  "effective_tflops": dense_flops * args.steps * world / td / 1e12,
                  "sparse_speedup": value / dense_value},
        "also": also,
        "stack": stack,
        "variants": variants,
    }
    if world == 1:
        step_s, desc, cores, _ = cpu_sample(wl)
        line["cpu_baseline"] = {"value": tokens_per_step / step_s, "unit": UNIT, "cores": cores,
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)


def run_kernel_loop(args, wl, local_rank):
    """One library call of the step in a loop (for ncu captures and isolated timings)."""
    import torch

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    hp = make_sets(wl, 1, dev)[0][0]
    with torch.cuda.stream(stream):
        hp.score_step(stream)
        hp.perm_step(stream)
    hp.attn_step(stream)   # leaves the permuted Q, K, V in the workspace for attn_kernel
    fn = {"score": hp.score_step, "perm": hp.perm_step, "score_perm": hp.score_perm_step,
          "attn": hp.attn_step, "attn_kernel": hp.attn_kernel_step,
          "rcmlp": hp.mlp_step}[args.kernel_loop]
    for _ in range(args.warmup):
        fn(stream)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        fn(stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    print(json.dumps({"kernel_loop": args.kernel_loop, "workload": wl.name,
                      "avg_us_per_call": 1e3 * ev0.elapsed_time(ev1) / args.steps,
                      "note": "inputs stay resident in L2 across calls"}), flush=True)


VITL_STACK = {"batch": 8, "grid": 64, "dim": 1024, "heads": 16, "head_dim": 64, "hidden": 4096,
              "blocks": 24, "global_blocks": (5, 11, 17, 23), "window": 14}


def stack_flops(cfg_pattern_g, cfg_pattern_w, K):
    """Algorithmic flops of one pass of the ViT-L stack: per block the qkv and proj GEMMs over its
    attention units' rows (pad rows of windowed blocks included: they are computed), the attention
    on its kept blocks and the MLP on the kept rows."""
    S = VITL_STACK
    B, C, Hd, T = S["batch"], S["dim"], S["hidden"], S["grid"] ** 2
    total = 0.0
    for i in range(S["blocks"]):
        pat = cfg_pattern_g if i in S["global_blocks"] else cfg_pattern_w
        rows = pat.units * pat.unit_tokens
        total += 2.0 * rows * C * 3 * C + 2.0 * rows * C * C
        total += workloads.attn_flops(pat.units, pat.unit_tokens, S["heads"], S["head_dim"], pat.rho)
        total += workloads.mlp_flops(B * K, C, Hd)
    return total, B * T


def measure_stack(args, dev, stream, densities, steps, warmup):
    """The ViT-L encoder stack through sparsesam_encoder_stack (24 full blocks: LN, qkv, attention,
    proj, LN2 + RC-MLP; global at 5, 11, 17, 23, the rest 14x14 windowed; 8 images of 64x64 tokens;
    one ranking of the tokens per pass) at each density: random-init weights drawn on the device,
    x updated in place pass after pass (each pass streams 0.6 GB of weights, well over L2)."""
    import torch

    from structured_activation_sparsity_b200 import _lib as L

    S = VITL_STACK
    B, G, C, Hd = S["batch"], S["grid"], S["dim"], S["hidden"]
    flags = [i in S["global_blocks"] for i in range(S["blocks"])]
    bf16_peak = peaks()[0]
    out = []
    for d in densities:
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(4)

        def rnd(*shape, scale=1.0, shift=0.0):
            t_ = torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)
            return (t_ * scale + shift).to(torch.bfloat16)
        blocks = []
        for _ in range(S["blocks"]):
            blocks.append({
                "ln1_w": rnd(C, scale=0.1, shift=1.0), "ln1_b": rnd(C, scale=0.1),
                "w_qkv": rnd(3 * C, C, scale=C ** -0.5), "b_qkv": rnd(3 * C, scale=0.1),
                "w_proj": rnd(C, C, scale=C ** -0.5), "b_proj": rnd(C, scale=0.1),
                "ln2_w": rnd(C, scale=0.1, shift=1.0), "ln2_b": rnd(C, scale=0.1),
                "w1": rnd(Hd, C, scale=C ** -0.5), "b1": rnd(Hd, scale=0.1),
                "w2": rnd(C, Hd, scale=Hd ** -0.5), "b2": rnd(C, scale=0.1)})
        weight_bytes = torch.cuda.memory_allocated(dev) - base
        wts = [L.block_weights(b) for b in blocks]
        x = rnd(B, G * G, C)
        lum = torch.rand(B, G, G, generator=gen, device=dev, dtype=torch.float32)
        cfg = L.make_cfg(B, G, G, "global", S["window"], S["heads"], S["head_dim"], d)
        wsb = L.sparsesam_encoder_stack_workspace(cfg, C, Hd)
        ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)

        def one():
            L.sparsesam_encoder_stack(cfg, lum, x, C, Hd, wts, flags, ws, wsb, stream)

        with torch.cuda.stream(stream):
            for _ in range(warmup):
                one()
        torch.cuda.synchronize()
        n0 = L.sparsesam_launch_count()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                one()
        ev1.record(stream)
        torch.cuda.synchronize()
        launches = (L.sparsesam_launch_count() - n0) // steps
        t = ev0.elapsed_time(ev1) / 1e3 / steps
        peak = torch.cuda.max_memory_allocated(dev) - base
        # one traced pass: each launch's CUDA-event time, summed per kernel over the pass
        L.sparsesam_trace_start(4096)
        with torch.cuda.stream(stream):
            one()
        recs = L.sparsesam_trace_stop()
        per = {}
        for name, ms in recs:
            per[name] = per.get(name, 0.0) + ms * 1e3
        if L.sparsesam_device_status(stream) != L.SS_OK:
            raise RuntimeError("a device wait timed out during the stack")
        pg = L.sparsesam_pattern(cfg)
        pw = L.sparsesam_pattern(L.make_cfg(B, G, G, "window", S["window"], S["heads"],
                                            S["head_dim"], d))
        flops, tokens = stack_flops(pg, pw, pg.keep)
        out.append({"density": d, "ms_per_stack": t * 1e3, "tokens_per_s": tokens / t,
                    "tokens_per_s_per_block": tokens * S["blocks"] / t,
                    "effective_tflops": flops / t / 1e12,
                    "frac_bf16_peak": flops / t / 1e12 / bf16_peak,
                    "global_rho": pg.rho, "window_rho": pw.rho, "kept_tokens_per_image": pg.keep,
                    "gpu_launches_per_stack": int(launches),
                    "peak_memory_bytes": int(peak), "weight_bytes": int(weight_bytes),
                    "workspace_bytes": int(wsb),
                    "traced_us_per_kernel": {k: round(v, 1) for k, v in
                                             sorted(per.items(), key=lambda kv: -kv[1])},
                    "steps": steps, "warmup": warmup})
        del blocks, wts, x, lum, ws
    torch.cuda.empty_cache()
    return out


def measure_variants(args, dev, stream, steps, warmup):
    """Attention-only timings of the variants, each over rotating input sets (> 3x L2 in total):
    Stripe-Sort attention with SAM's relative-position bias (ViT-B global and windowed shapes),
    the PE-style partial attention with 2-D RoPE (PE-Core-L14-336: 128 images of 1 class token +
    24 x 24 patches, 16 heads x 64, density 0.5), and plain attention only (the attention-only
    registry variant) on the ViT-B global block. Per call: CUDA events around `steps` calls."""
    import torch

    from structured_activation_sparsity_b200 import _lib as L

    bf16_peak = peaks()[0]
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)

    def bf(*shape, scale=1.0):
        return (torch.randn(*shape, generator=gen, device=dev) * scale).to(torch.bfloat16)

    def perm_of(cfg, U, N):
        lum = torch.rand(cfg.batch, cfg.grid_h, cfg.grid_w, generator=gen, device=dev)
        score = torch.empty(cfg.batch, cfg.grid_h * cfg.grid_w, dtype=torch.float64, device=dev)
        perm = torch.empty(U, N, dtype=torch.int32, device=dev)
        L.sparsesam_score_perm(cfg, lum, score, perm, None, None, stream)
        return perm

    def timed(calls):
        with torch.cuda.stream(stream):
            for i in range(warmup):
                calls[i % len(calls)]()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        with torch.cuda.stream(stream):
            for i in range(steps):
                calls[i % len(calls)]()
        ev1.record(stream)
        torch.cuda.synchronize()
        if L.sparsesam_device_status(stream) != L.SS_OK:
            raise RuntimeError("a device wait timed out in a variant")
        t = ev0.elapsed_time(ev1) / 1e3 / steps
        L.sparsesam_trace_start(64)    # one traced call: each launch's CUDA-event time
        with torch.cuda.stream(stream):
            calls[0]()
        per = {}
        for n_, ms in L.sparsesam_trace_stop():
            per[n_] = round(per.get(n_, 0.0) + ms * 1e3, 1)
        traced[0] = per
        return t

    out = {}
    traced = [None]
    for name, wl_name in (("relpos_vitb_global", "vitb_global"), ("relpos_vitb_window", "vitb_window"),
                          ("attn_only_vitb_global", "vitb_global")):
        wl = workloads.get(wl_name)
        cfg = L.cfg_for(wl)
        U, N = wl.units, wl.unit_tokens
        pat = L.sparsesam_pattern(cfg)
        Hu, Wu = (wl.window, wl.window) if wl.mode == "window" else (wl.grid_h, wl.grid_w)
        relpos = name.startswith("relpos")
        wsb = (L.sparsesam_attn_relpos_workspace(cfg) if relpos else L.sparsesam_attn_workspace(cfg))
        per_set = 4 * U * N * wl.heads * wl.head_dim * 2 + wsb
        n_sets = max(2, math.ceil(3 * L2_BYTES / per_set))
        calls = []
        for _ in range(n_sets):
            q, k, v, o = (bf(U, N, wl.heads, wl.head_dim) for _ in range(4))
            perm = perm_of(cfg, U, N)
            ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
            if relpos:
                rh, rw = bf(2 * Hu - 1, wl.head_dim, scale=0.1), bf(2 * Wu - 1, wl.head_dim, scale=0.1)
                calls.append(lambda q=q, k=k, v=v, o=o, perm=perm, ws=ws, rh=rh, rw=rw:
                             L.sparsesam_attn_relpos(cfg, q, k, v, perm, rh, rw, o, ws, wsb, stream))
            else:
                calls.append(lambda q=q, k=k, v=v, o=o, perm=perm, ws=ws:
                             L.sparsesam_attn(cfg, q, k, v, perm, o, ws, wsb, stream))
        t = timed(calls)
        flops = workloads.attn_flops(U, N, wl.heads, wl.head_dim, pat.rho)
        out[name] = {"us_per_call": t * 1e6, "tokens_per_s": wl.batch * wl.tokens_per_image / t,
                     "attn_tflops": flops / t / 1e12, "frac_bf16_peak": flops / t / 1e12 / bf16_peak,
                     "traced_us": traced[0],
                     "note": "gather + (bias GEMM) + attention + un-permute per call"}
        del calls
        torch.cuda.empty_cache()
    # PE-Core-L14-336 partial attention with RoPE
    B, G, P_, H, D, d = 128, 24, 1, 16, 64, 0.5
    cfg = L.make_cfg(B, G, G, "global", 14, H, D, d)
    pat = L.sparsesam_pattern(cfg)
    wsb = L.sparsesam_attn_partial_workspace(cfg, P_)
    NT = P_ + G * G
    calls = []
    n_sets = max(2, math.ceil(3 * L2_BYTES / (4 * B * NT * H * D * 2 + wsb)))
    for _ in range(n_sets):
        q, k, v, o = (bf(B, NT, H, D) for _ in range(4))
        perm = perm_of(cfg, B, G * G)
        ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
        calls.append(lambda q=q, k=k, v=v, o=o, perm=perm, ws=ws:
                     L.sparsesam_attn_partial(cfg, P_, 10000.0, q, k, v, perm, o, ws, wsb, stream))
    t = timed(calls)
    flops = workloads.attn_flops(B, G * G, H, D, pat.rho) + 4.0 * B * H * D * (
        2 * P_ * NT - P_ * P_)   # prefix rows and the prefix keys of the patch rows
    out["partial_pe_core_l14_336"] = {
        "us_per_call": t * 1e6, "tokens_per_s": B * NT / t, "attn_tflops": flops / t / 1e12,
        "frac_bf16_peak": flops / t / 1e12 / bf16_peak,
        "config": {"images": B, "prefix": P_, "grid": f"{G}x{G}", "heads": H, "head_dim": D,
                   "density": d, "rope_base": 10000.0, "realised_density": pat.rho},
        "traced_us": traced[0],
        "note": "RoPE gather + attention + prefix merge + prefix rows per call"}
    del calls
    torch.cuda.empty_cache()
    return out


def run_stack(args, local_rank):
    """The ViT-L stack alone at the density sweep, one JSON line per density (no bench line)."""
    import torch

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    for r in measure_stack(args, dev, stream, (1.0, 0.5, 0.4, 0.3), args.steps, args.warmup):
        print(json.dumps({"stack": "vitl_24_blocks", **r}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="vith_global", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--also", default="vitb_global,vitb_window",
                    help="other workloads measured the same way, reported under 'also' "
                         "(comma-separated; empty for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel-loop", default=None,
                    choices=["score", "perm", "score_perm", "attn", "attn_kernel", "rcmlp"],
                    help="run only this library call in a loop (profiling aid; no bench line)")
    ap.add_argument("--stack", action="store_true",
                    help="time the ViT-L 24-block stack at densities 1.0/0.5/0.4/0.3 (no bench line)")
    ap.add_argument("--no-stack", action="store_true",
                    help="leave the ViT-L stack sweep and the variants out of the bench line")
    ap.add_argument("--variants", action="store_true",
                    help="time the attention variants only (no bench line)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    wl = workloads.get(args.workload)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    if args.kernel_loop:
        run_kernel_loop(args, wl, local_rank)
        return
    if args.stack:
        run_stack(args, local_rank)
        return
    if args.variants:
        import torch
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        print(json.dumps(measure_variants(args, dev, torch.cuda.Stream(device=dev), args.steps,
                                          args.warmup)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
    try:
        run_ours(args, wl, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
