#!/usr/bin/env python
"""Paged decode step benchmark (B200, sm_100a).

One step = the whole decode hot path over one batch: copy_blocks for pending
copy-on-write pairs (none in the llama7b batch), then the new token of every
sequence written into its slot and the attention over the updated cache.  By
default both happen in one paged_attention_decode_append launch (plus the
split-K merge when the workload splits); --step separate runs reshape_and_cache
and paged_attention_decode instead.  The default workload is the Llama-2-7B-shaped batch:
256 sequences, 32 = 32 heads, head_dim 128, block_size 16, contexts uniform in
[500, 1524], 32768-block pool.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama7b|gqa|bs_sweep_8|...] [--step fused|separate]

Prints ONE JSON line (rank 0).  value = K+V bytes the attention reads per step,
summed over ranks, divided by the device time of the K timed steps (max over
ranks).  Multi-GPU runs are independent replicas of the batch on every rank
(weak scaling, no collective on the data path).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged decode attention KV GB/s (% of B200 HBM peak) and decode tokens/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
# The nominal B200 HBM3e bandwidth (~8 TB/s) the target is stated against; the roofline
# fractions use the measured copy bandwidth instead (a read-only stream can exceed a copy).
NOMINAL_HBM_GBS = 8000.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--step", choices=["fused", "separate", "shared"], default="fused",
                    help="fused: one paged_attention_decode_append call writes the new tokens "
                         "and attends; separate: reshape_and_cache then paged_attention_decode; "
                         "shared (cow workload): the fused shared-prefix call, which reads each "
                         "group's shared prompt blocks once")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=1,
                    help="attention layers per decode step, each with its own pools (a copy of "
                         "the workload's), run as one CUDA graph (LayeredDecodeStep)")
    ap.add_argument("--partition-size", type=int, default=None,
                    help="split-K partition size (default: the workload's)")
    ap.add_argument("--no-sub-results", action="store_true",
                    help="default llama7b run: skip the other workloads' lines (block-size sweep, "
                         "gqa, cow shared-prefix step)")
    ap.add_argument("--sub-steps", type=int, default=300,
                    help="timed steps of each sub-result workload")
    ap.add_argument("--eager", action="store_true",
                    help="cow workload: launch every step from Python instead of replaying "
                         "one CUDA graph per step")
    return ap.parse_args(argv)


# ---- distributed plumbing -----------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(backend, world, device_index=None):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl" and device_index is not None:
            import torch
            kw["device_id"] = torch.device("cuda", device_index)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)


def barrier(world, device_index=None):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device_index])
        else:
            dist.barrier()


def aggregate(ms: float, units: float, world: int, device=None):
    """(max over ranks of the timed ms, sum over ranks of the units processed)."""
    if world == 1:
        return ms, units
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ---- clocks --------------------------------------------------------------------------

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling of one GPU's clocks and throttle reasons (read-only)."""

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + CLOCK_FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        # samples under load: power above the midpoint of the observed range
        if power:
            cut = (min(power) + max(power)) / 2
            loaded = [num(r[1]) for r in rows if num(r[3]) is not None and num(r[3]) >= cut]
        else:
            loaded = sm
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded or sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


def gpu_id_for(device_index: int) -> str:
    import torch
    props = torch.cuda.get_device_properties(device_index)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        s = str(uuid)
        return s if s.startswith("GPU-") else "GPU-" + s
    return str(device_index)


# ---- peaks and ncu traffic -------------------------------------------------------------

def describe(w) -> str:
    """The workload string both arms put in config.workload."""
    lens = wl.context_lens(w)
    return ("%s: %d seqs, %d query / %d kv heads, head_dim %d, block_size %d, contexts %d..%d, "
            "%d-block pool" % (w.name, w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
                               w.block_size, lens.min(), lens.max(), w.num_blocks))


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(path: str) -> str:
    """sha256/16 of a kernel file together with the headers every kernel file includes."""
    h = hashlib.sha256()
    d = os.path.dirname(path)
    for f in (path, os.path.join(d, "common.cuh"), os.path.join(d, "kernels.h")):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this
    exact kernel source; None otherwise."""
    summary = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    src = os.path.join(ROOT, "paged_kv_cache_393_b200", "csrc", kernel_file)
    if not os.path.exists(summary) or not os.path.exists(src):
        return None
    h = kernel_source_hash(src)
    with open(summary) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel_file \
                    and parts[1] == h and parts[2] == workload:
                return float(parts[3])
    return None


# ---- the CUDA arm ------------------------------------------------------------------------

def time_decode(gb, part, step_kind, K, warmup, dev, stream, world, local):
    """Times K decode steps of a PagedBatch on `stream`: the fused append + attention call
    (step_kind "fused"), or reshape_and_cache then paged_attention_decode ("separate"),
    plus the split-K merge when the plan splits.  CUDA events bracket the attention call
    of every step; clocks are sampled over the timed region."""
    import torch

    import paged_kv_cache_393_b200 as pkv
    w = gb.w
    B, H, Hk, D = w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim
    need = pkv.paged_attention_workspace_bytes(B, H, Hk, D, w.block_size, gb.max_context_len, part)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
    # split-K (a merge kernel and partial bytes) only when the plan partitions the contexts;
    # the tensor-core path needs a workspace word even in a single pass
    pt = pkv.paged_attention_partition_tokens(B, H, Hk, D, w.block_size, gb.max_context_len, part)
    fused = step_kind == "fused"
    launches_per_step = (1 if fused else 2) + (1 if pt > 0 else 0)   # [reshape,] attention[, merge]
    G = H // Hk
    kernel_file = "attention_mma.cu" if (2 <= G <= 8 and w.block_size >= 8) else "attention_simt.cu"

    def attention():
        if fused:
            pkv.paged_attention_decode_append(gb.out, gb.q, gb.k_new, gb.v_new, gb.key_cache,
                                              gb.value_cache, gb.block_tables, gb.context_lens,
                                              w.scale, gb.max_context_len, part, ws, stream=stream)
        else:
            pkv.paged_attention_decode(gb.out, gb.q, gb.key_cache, gb.value_cache,
                                       gb.block_tables, gb.context_lens, w.scale,
                                       gb.max_context_len, part, ws, stream=stream)

    def cache_update():
        if not fused:
            pkv.reshape_and_cache(gb.k_new, gb.v_new, gb.key_cache, gb.value_cache, gb.slots,
                                  stream=stream)

    for _ in range(max(warmup, 3)):
        cache_update()
        attention()
    torch.cuda.synchronize(dev)
    pkv.device_errors(clear=True)

    ev_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    # keep the GPU busy while the sampler spins up, then time exactly K steps
    for _ in range(20):
        cache_update()
        attention()
    barrier(world, local)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for i in range(K):
        cache_update()
        ev_a[i][0].record(stream)
        attention()
        ev_a[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, local)
    clocks = sampler.stop()
    flags = pkv.device_errors(clear=True)
    if flags:
        raise SystemExit("device error flags %#x during the timed steps (%s)" % (flags, w.name))

    per_launch = sorted(a.elapsed_time(b) for a, b in ev_a)
    attn_ms = sum(per_launch) / K
    attn_median_ms = per_launch[K // 2] if K % 2 else 0.5 * (per_launch[K // 2 - 1] +
                                                             per_launch[K // 2])
    kv_bytes = gb.kv_bytes()
    # the attention call's algorithmic bytes per launch: K+V rows read, q read, out
    # written, table entries and lengths read, new rows, split partials written and read
    nblk = (gb.lens_host + w.block_size - 1) // w.block_size
    attn_bytes = kv_bytes + 2 * B * H * D * 2 + int(nblk.sum()) * 4 + B * 4
    if fused:
        attn_bytes += 2 * B * Hk * D * 2 * 2
    # (the split-K partials are the implementation's own traffic, not the method's: they
    # are reported apart and left out of the algorithmic bytes)
    partial_bytes = 0
    if pt > 0:
        parts = (gb.lens_host + pt - 1) // pt
        partial_bytes = int(parts[parts > 1].sum()) * H * (D + 2) * 4 * 2
    return {"ms_total": t0.elapsed_time(t1), "K": K, "attn_ms": attn_ms,
            "attn_median_ms": attn_median_ms, "kv_bytes": kv_bytes,
            "attn_bytes": attn_bytes, "partial_bytes": partial_bytes,
            "launches": K * launches_per_step, "clocks": clocks, "kernel_file": kernel_file,
            "partition_tokens": pt}


def roofline_of(res, workload):
    peak, peak_kind = hbm_peak()
    achieved = res["attn_bytes"] / (res["attn_ms"] / 1e3) / 1e9
    return {"bound": "hbm", "kernel": res["kernel_file"].replace(".cu", ""),
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "traffic": recorded_traffic(res["kernel_file"], workload),
            "algorithmic_bytes": res["attn_bytes"], "split_partial_bytes": res["partial_bytes"],
            "avg_launch_ms": round(res["attn_ms"], 5),
            "median_launch_ms": round(res["attn_median_ms"], 5)}


def sub_entry(w, res, step_kind):
    """One sub-result: a workload's own device-timed line (K+V GB/s, its roofline, clocks)."""
    ms = res["ms_total"] / res["K"]
    return {"workload": describe(w), "step": step_kind, "steps": res["K"],
            "ms_per_step": round(ms, 5),
            "value": round(res["kv_bytes"] / (ms / 1e3) / 1e9, 2), "unit": UNIT,
            "tokens_per_s": round(w.num_seqs / (ms / 1e3), 1),
            "pct_of_hbm_peak": round(100 * res["kv_bytes"] / (ms / 1e3) / 1e9 / NOMINAL_HBM_GBS, 2),
            "partition_tokens": res["partition_tokens"],
            "roofline": roofline_of(res, w.name), "gpu_launches": res["launches"],
            "clocks": res["clocks"]}


def run_ours(args):
    import torch

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist("nccl", world, local)
    dev = torch.device("cuda", local)
    import paged_kv_cache_393_b200 as pkv
    from batches import PagedBatch, paged_batches
    pkv.load_library()
    w = wl.get(args.workload)
    if w.lens == "cow":
        line = measure_cow(args, w, dev, world, rank, local, args.step, args.steps,
                           min(args.e2e_steps, w.decode_steps, 50))
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.layers > 1:
        return run_layers(args, w, dev, world, rank, local)
    # the default run also reports the other workloads (sub_results) on one GPU
    subs = args.workload == "llama7b" and world == 1 and not args.no_sub_results
    if subs:
        # block-size sweep: the llama7b tokens and values at block sizes 8/16/32/64, drawn once
        sweep = paged_batches([wl.bs_sweep(8), w, wl.bs_sweep(32), wl.bs_sweep(64)], dev)
        gb = sweep[1]
    else:
        sweep = []
        gb = PagedBatch(w, dev)
    part = w.partition_size if args.partition_size is None else args.partition_size
    B, H, Hk, D = w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim
    stream = torch.cuda.Stream(dev)
    K = args.steps
    res = time_decode(gb, part, args.step, K, args.warmup, dev, stream, world, local)
    kv_bytes = res["kv_bytes"]
    ms_max, kv_all = aggregate(res["ms_total"], float(kv_bytes) * K, world, dev)
    ms_per_step = ms_max / K
    value = kv_all / (ms_max / 1e3) / 1e9

    # end to end through the public API: host buffers in, host result out
    e2e = None
    if args.e2e_steps > 0:
        # paged_decode_step_host: the inputs uploaded from pinned host memory, the fused
        # append + attention, the output downloaded, all in one C call per step
        sess = pkv.DecodeSession(gb.key_cache, gb.value_cache, B, H, gb.max_blocks,
                                 gb.max_context_len, w.scale, part)
        pin = lambda a: torch.from_numpy(a).pin_memory()  # noqa: E731
        hq, hk, hv = pin(gb.q_host), pin(gb.k_new_host), pin(gb.v_new_host)
        ht, hl = pin(gb.tables_host), pin(gb.lens_host)
        hout = torch.empty((B, H, D), dtype=torch.float16).pin_memory()
        for _ in range(5):
            sess.step(hq, hk, hv, ht, hl, hout, stream=stream)
        torch.cuda.synchronize(dev)
        barrier(world, local)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        E = args.e2e_steps
        e0.record(stream)
        for _ in range(E):
            sess.step(hq, hk, hv, ht, hl, hout, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms, e_bytes = aggregate(e0.elapsed_time(e1), float(kv_bytes) * E, world, dev)
        e2e = {"value": round(e_bytes / (e_ms / 1e3) / 1e9, 2), "unit": UNIT,
               "ms_per_step": round(e_ms / E, 4), "call": "paged_decode_step_host",
               "h2d_bytes_per_step": sess.h2d_bytes(), "d2h_bytes_per_step": sess.d2h_bytes()}
        del sess

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    sub_results = None
    if subs:
        KS = max(args.sub_steps, 3)
        sub_results = []
        for g in sweep:
            r = res if g is gb and K >= KS else time_decode(g, part, args.step, KS, args.warmup,
                                                              dev, stream, world, local)
            sub_results.append(sub_entry(g.w, r, args.step))
        del g, sweep, gb
        torch.cuda.empty_cache()
        gq = PagedBatch(wl.get("gqa"), dev)
        r = time_decode(gq, gq.w.partition_size, args.step, KS, args.warmup, dev, stream, world,
                        local)
        sub_results.append(sub_entry(gq.w, r, args.step))
        del gq, r
        torch.cuda.empty_cache()
        cow = measure_cow(args, wl.get("cow"), dev, world, rank, local, "shared",
                          max(KS, 200), 0)
        sub_results.append({k: cow[k] for k in (
            "workload", "step", "steps", "ms_per_step", "value", "unit", "tokens_per_s",
            "unique_kv_GB_per_s", "roofline", "copy_blocks", "gpu_launches", "clocks")})
        torch.cuda.empty_cache()

    if rank == 0:
        peak, _ = hbm_peak()
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "accumulate": "f32", "data": "synthetic",
            "config": {
                "workload": describe(w),
                "seed": w.seed, "partition_size": part, "kv_bytes_per_step": kv_bytes,
                "step": args.step,
                "l2": "no flush: each step reads %.2f GB of K/V, far above the 126 MB L2"
                      % (kv_bytes / 1e9),
                "parallelism": "replicas x%d" % world},
            "tokens_per_s": round(B * world / (ms_per_step / 1e3), 1),
            "steps_per_s": round(1e3 / ms_per_step, 2),
            "roofline": roofline_of(res, args.workload),
            "pct_of_hbm_peak": round(100 * value / world / NOMINAL_HBM_GBS, 2),
            "hbm_peak_nominal_gbs": NOMINAL_HBM_GBS,
            "pct_of_measured_copy_peak": round(100 * value / world / peak, 2),
            "gpu_launches": res["launches"],
            "clocks": res["clocks"],
            "e2e": e2e,
            "cpu_baseline": cpu,
            "sub_results": sub_results,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_layers(args, w, dev, world, rank, local):
    """A decode step over args.layers attention layers (every layer its own pools, here copies
    of the workload's), each layer's fused append + attention, replayed as one CUDA graph;
    the same launches issued eagerly from Python are timed too."""
    import torch

    import paged_kv_cache_393_b200 as pkv
    from batches import PagedBatch
    gb = PagedBatch(w, dev)
    Lyr = args.layers
    pool_bytes = 2 * gb.key_cache.numel() * 2
    free, _ = torch.cuda.mem_get_info(dev)
    if pool_bytes * (Lyr - 1) > 0.85 * free:
        raise SystemExit("%d layers need %.1f GB of pools, %.1f GB free: use fewer layers or a "
                         "smaller workload" % (Lyr, pool_bytes * Lyr / 1e9, free / 1e9))
    kcs, vcs = [gb.key_cache], [gb.value_cache]
    for _ in range(Lyr - 1):
        kcs.append(gb.key_cache.clone())
        vcs.append(gb.value_cache.clone())
    part = w.partition_size if args.partition_size is None else args.partition_size
    B, H, Hk, D = w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim
    stream = torch.cuda.Stream(dev)
    step = pkv.LayeredDecodeStep(kcs, vcs, B, H, gb.max_blocks, gb.max_context_len, w.scale, part,
                                 stream=stream)
    step.set_inputs(q=gb.q.expand(Lyr, -1, -1, -1), k_new=gb.k_new.expand(Lyr, -1, -1, -1),
                    v_new=gb.v_new.expand(Lyr, -1, -1, -1), block_tables=gb.block_tables,
                    context_lens=gb.context_lens)
    need = pkv.paged_attention_workspace_bytes(B, H, Hk, D, w.block_size, gb.max_context_len, part)
    launches_per_step = Lyr * (1 + (1 if need > 0 else 0))

    def timed(K, fn):
        for _ in range(max(args.warmup, 3)):
            fn()
        barrier(world, local)
        torch.cuda.synchronize(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(K):
            fn()
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, local)
        return t0.elapsed_time(t1)

    eager_ms = timed(max(args.steps // 4, 3), step.replay) / max(args.steps // 4, 3)
    step.capture()
    pkv.device_errors(clear=True)
    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    K = args.steps
    ms_total = timed(K, step.replay)
    clocks = sampler.stop()
    flags = pkv.device_errors(clear=True)
    if flags:
        raise SystemExit("device error flags %#x during the timed steps" % flags)
    kv_bytes = gb.kv_bytes() * Lyr
    ms_max, kv_all = aggregate(ms_total, float(kv_bytes) * K, world, dev)
    ms_per_step = ms_max / K
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": round(kv_all / (ms_max / 1e3) / 1e9, 2), "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "accumulate": "f32", "data": "synthetic",
            "config": {"workload": "%s x %d layers (every layer its own pools), one CUDA graph "
                                   "per step" % (w.name, Lyr),
                       "seed": w.seed, "partition_size": part, "layers": Lyr,
                       "kv_bytes_per_step": kv_bytes, "parallelism": "replicas x%d" % world},
            "tokens_per_s": round(B * world / (ms_per_step / 1e3), 1),
            "us_per_layer": round(ms_per_step * 1e3 / Lyr, 2),
            "eager_ms_per_step": round(eager_ms, 5),
            "gpu_launches": K * launches_per_step, "clocks": clocks, "e2e": None,
            "cpu_baseline": None,
        }), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def measure_cow(args, w, dev, world, rank, local, step_kind, K, e2e_steps):
    """The copy-on-write workload: 32 prompts of 1000 tokens forked into 8 samples,
    then decode steps.  Step 0 copies the 224 shared partial tail blocks
    (copy_blocks) before its scatter and attention; the steps are replayed in
    order.  Replays do the same work; their cache contents may differ (a replayed
    step-0 copy overwrites later rows of the copied blocks), which the timing
    does not depend on.  Returns the workload's JSON line (a dict)."""
    import numpy as np
    import torch

    import paged_kv_cache_393_b200 as pkv
    from batches import CowBatch
    gb = CowBatch(w, dev)
    B, H, Hk, D = w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim
    steps_host = [gb.prepare_step() for _ in range(w.decode_steps)]
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    shared = step_kind == "shared"
    steps = []
    unique_total = 0
    for h in steps_host:
        st = dict(q=up(h["q"]), k=up(h["k"]), v=up(h["v"]), slots=up(h["slots"]),
                  tables=up(h["tables"]), lens=up(h["lens"]),
                  pairs=up(h["pairs"]) if len(h["pairs"]) else None,
                  kv_bytes=int(h["lens"].astype(np.int64).sum()) * wl.kv_bytes_per_token(Hk, D))
        if shared:
            pre, groups = pkv.prefix_groups(h["tables"], h["lens"], w.block_size, 8 // (H // Hk))
            st["pre"], st["groups"] = up(pre), up(groups)
            st["max_prefix"] = int(groups[:, 0].max()) * w.block_size if len(groups) else 0
            st["max_suffix"] = int((h["lens"] - pre).max())
            # K/V bytes the shared-prefix call reads: each group's prefix once, the rest per sequence
            uniq = int((h["lens"] - pre).astype(np.int64).sum()) + int(groups[:, 0].sum()) * w.block_size
            st["unique_bytes"] = uniq * wl.kv_bytes_per_token(Hk, D)
        steps.append(st)
    out = torch.empty((B, H, D), dtype=torch.float16, device=dev)
    cpart = 0 if args.partition_size is None else args.partition_size
    if shared:
        need = pkv.paged_attention_shared_prefix_workspace_bytes(B, H, Hk, D, w.block_size,
                                                                 gb.max_context_len, cpart)
    else:
        need = pkv.paged_attention_workspace_bytes(B, H, Hk, D, w.block_size, gb.max_context_len,
                                                   cpart)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
    plain_split = pkv.paged_attention_partition_tokens(B, H, Hk, D, w.block_size,
                                                       gb.max_context_len, cpart) > 0
    stream = torch.cuda.Stream(dev)
    n_pairs = len(steps_host[0]["pairs"])
    copy_bytes = 2 * n_pairs * 2 * Hk * w.block_size * D * 2   # K and V blocks read + written

    def run_step(j, ev=None):
        st = steps[j]
        if st["pairs"] is not None:
            if ev is not None:
                ev[0].record(stream)
            pkv.copy_blocks([gb.key_cache], [gb.value_cache], st["pairs"], stream=stream)
            if ev is not None:
                ev[1].record(stream)
        if shared:
            pkv.paged_attention_decode_shared_prefix(
                out, st["q"], gb.key_cache, gb.value_cache, st["tables"], st["lens"], st["pre"],
                st["groups"], w.scale, gb.max_context_len, cpart, ws, k_new=st["k"], v_new=st["v"],
                stream=stream, max_prefix_tokens=st["max_prefix"],
                max_suffix_tokens=st["max_suffix"])
        elif step_kind == "fused":
            pkv.paged_attention_decode_append(out, st["q"], st["k"], st["v"], gb.key_cache,
                                              gb.value_cache, st["tables"], st["lens"], w.scale,
                                              gb.max_context_len, cpart, ws, stream=stream)
        else:
            pkv.reshape_and_cache(st["k"], st["v"], gb.key_cache, gb.value_cache, st["slots"],
                                  stream=stream)
            pkv.paged_attention_decode(out, st["q"], gb.key_cache, gb.value_cache, st["tables"],
                                       st["lens"], w.scale, gb.max_context_len, cpart, ws,
                                       stream=stream)

    for j in range(w.decode_steps):   # first pass: the steps in order
        run_step(j)
    for j in range(max(args.warmup, 3)):
        run_step(j % w.decode_steps)
    torch.cuda.synchronize(dev)
    pkv.device_errors(clear=True)
    # the copy-on-write step alone, timed with events around eager launches
    copy_ev = []
    if steps[0]["pairs"] is not None:
        for _ in range(20):
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(stream)
            pkv.copy_blocks([gb.key_cache], [gb.value_cache], steps[0]["pairs"], stream=stream)
            ev[1].record(stream)
            copy_ev.append(ev)
    # One CUDA graph per step (the same launches, replayed without Python in the way)
    graphs = None
    if not args.eager:
        graphs = []
        for j in range(w.decode_steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run_step(j)
            graphs.append(g)
        torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()

    def replay(j):
        if graphs is None:
            run_step(j)
        else:
            with torch.cuda.stream(stream):   # a graph launches on the current stream
                graphs[j].replay()

    for j in range(20):
        replay(j % w.decode_steps)
    barrier(world, local)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    kv_total = 0
    launches = 0
    copies_total = 0
    h0 = time.perf_counter()
    for i in range(K):
        j = i % w.decode_steps
        if steps[j]["pairs"] is not None:
            launches += 1
            copies_total += copy_bytes
        replay(j)
        if shared:
            # prefix pass (when there are groups), suffix pass, merge (unless every suffix
            # fits one partition: then the suffix pass finishes the outputs)
            pt = cpart if cpart > 0 else 512
            launches += (1 if steps[j]["max_prefix"] > 0 else 0) + 1 + \
                (1 if steps[j]["max_suffix"] > pt else 0)
        else:
            # [reshape,] attention, and the merge when the plan splits
            launches += {"fused": 1, "separate": 2}[step_kind] + (1 if plain_split else 0)
        kv_total += steps[j]["kv_bytes"]
        unique_total += steps[j].get("unique_bytes", 0)
    host_ms = (time.perf_counter() - h0) * 1e3
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, local)
    clocks = sampler.stop()
    flags = pkv.device_errors(clear=True)
    if flags:
        raise SystemExit("device error flags %#x during the timed steps" % flags)
    ms_max, kv_all = aggregate(t0.elapsed_time(t1), float(kv_total), world, dev)
    ms_per_step = ms_max / K
    copy_us = (sum(a.elapsed_time(b) for a, b in copy_ev) / len(copy_ev) * 1e3) if copy_ev else None
    prefix_blocks = w.prompts * (w.prompt_len // w.block_size)

    # end to end through DecodeSession (host buffers in, host output back), the steps in order
    # from the start (copy-on-write pairs at step 0); the host grouping of the shared-prefix
    # step is inside the timed region
    e2e = None
    E = min(e2e_steps, w.decode_steps)
    if E > 0:
        sess = pkv.DecodeSession(gb.key_cache, gb.value_cache, B, H, gb.max_blocks,
                                 gb.max_context_len, w.scale, cpart, max_pairs=max(n_pairs, 1),
                                 shared_prefix=shared)
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()  # noqa: E731
        hs = [{k: pin(steps_host[j][k]) for k in ("q", "k", "v", "tables", "lens")}
              for j in range(E)]
        hpairs = pin(steps_host[0]["pairs"]) if n_pairs else None
        hout = torch.empty((B, H, D), dtype=torch.float16).pin_memory()

        def e2e_step(j):
            h = hs[j]
            sess.step(h["q"], h["k"], h["v"], h["tables"], h["lens"], hout,
                      pairs=hpairs if j == 0 else None, stream=stream)

        for j in range(min(3, E)):
            e2e_step(j)
        torch.cuda.synchronize(dev)
        barrier(world, local)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d = 0
        for j in range(E):
            e2e_step(j)
            h2d += sess.h2d_bytes()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms, e_bytes = aggregate(e0.elapsed_time(e1),
                                  float(sum(steps[j]["kv_bytes"] for j in range(E))), world, dev)
        e2e = {"value": round(e_bytes / (e_ms / 1e3) / 1e9, 2), "unit": UNIT,
               "ms_per_step": round(e_ms / E, 4), "steps": E, "call": "paged_decode_step_host",
               "h2d_bytes_per_step": int(h2d / E), "d2h_bytes_per_step": sess.d2h_bytes()}
    peak, peak_kind = hbm_peak()
    # roofline of the step: the K/V bytes it must read (with shared prefixes: each group's
    # prefix once) plus the copy-on-write copies, over the device time
    alg = (unique_total if shared else kv_total) + copies_total
    achieved = alg * world / (ms_max / 1e3) / 1e9
    return {
            "metric": METRIC, "value": round(kv_all / (ms_max / 1e3) / 1e9, 2), "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "accumulate": "f32", "data": "synthetic",
            "config": {"workload": "cow: %d prompts x %d tokens forked into %d samples, %d decode "
                                   "steps replayed in order; K/V bytes counted per sample "
                                   "(shared prefix blocks counted once per reader)" % (
                                       w.prompts, w.prompt_len, w.samples, w.decode_steps),
                       "seed": w.seed, "step": step_kind, "partition_size": cpart,
                       "l2": "no flush; shared prefix blocks (%d x 128 KiB x 2) "
                             "can hit in L2" % prefix_blocks,
                       "parallelism": "replicas x%d" % world},
            "tokens_per_s": round(B * world / (ms_per_step / 1e3), 1),
            "unique_kv_GB_per_s": round(unique_total * world / (ms_max / 1e3) / 1e9, 2)
            if shared else None,
            "copy_blocks": {"pairs": n_pairs, "bytes": copy_bytes, "avg_us": copy_us,
                            "GB_per_s": round(copy_bytes / (copy_us / 1e6) / 1e9, 1) if copy_us else None,
                            "peak": peak, "peak_kind": peak_kind},
            "roofline": {"bound": "hbm",
                         "kernel": "mma_prefix + suffix pass" if shared else "attention_simt",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                         "traffic": None, "algorithmic_bytes": int(alg / K),
                         "scope": "whole step (device time per step), K/V bytes read once "
                                  "per group prefix plus the copy-on-write copies"},
            "step": step_kind, "workload": "cow (%d prompts x %d tokens, %d samples each)" % (
                w.prompts, w.prompt_len, w.samples),
            "gpu_launches": launches, "clocks": clocks, "e2e": e2e, "cpu_baseline": None,
            "launch": "eager" if graphs is None else "one CUDA graph per step",
            "host_issue_ms_per_step": round(host_ms / K, 4),
    }


# ---- the oracle: cpu_baseline leg and reference arm ---------------------------------------

def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_sample(w, seconds, cores):
    """Largest prefix of the batch whose oracle attention takes about `seconds`."""
    from oracle.batch import OracleBatch
    probe = OracleBatch(w, sample=[0, 1])
    t = time.perf_counter()
    probe.attention(nthreads=cores)
    per_seq = max((time.perf_counter() - t) / 2, 1e-4)
    n = int(max(2, min(w.num_seqs, seconds / per_seq)))
    return OracleBatch(w, sample=list(range(n)))


def cpu_baseline(w, seconds):
    cores = _cores()
    ob = _oracle_sample(w, seconds, cores)
    t = time.perf_counter()
    ob.attention(nthreads=cores)
    dt = time.perf_counter() - t
    kv = int(ob.lens.astype("int64").sum()) * wl.kv_bytes_per_token(w.num_kv_heads, w.head_dim)
    return {"value": round(kv / dt / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%d of %d sequences (all %d heads, %d tokens) of the %s batch; fp64 C "
                      "oracle on %d threads; %.1f s" % (len(ob.sample), w.num_seqs, w.num_heads,
                                                        int(ob.lens.sum()), w.name, cores, dt)}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import numpy as np

    import oracle
    w = wl.get(args.workload)
    cores = _cores()
    steps, warm = args.steps, max(args.warmup, 3)
    per_step = min(10.0, 150.0 / (steps + warm))
    ob = _oracle_sample(w, per_step, cores)
    bs = w.block_size
    tables = ob.compact_tables
    last = ob.lens - 1
    slots = np.array([tables[j, L // bs] * bs + L % bs for j, L in enumerate(last)], np.int64)
    kv_new = [wl.sequence_kv(w.seed, b, int(L) + 1, w.num_kv_heads, w.head_dim)
              for b, L in zip(ob.sample, last)]
    k_new = np.stack([k[-1] for k, _ in kv_new])
    v_new = np.stack([v[-1] for _, v in kv_new])

    def step():
        kc, vc = oracle.reshape_and_cache(ob.key_cache, ob.value_cache, k_new, v_new, slots, bs)
        return oracle.paged_attention(ob.q, kc, vc, tables, ob.lens, w.scale, bs, w.num_kv_heads,
                                      nthreads=cores)
    for _ in range(warm):
        step()
    t = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t) / steps
    kv = int(ob.lens.astype("int64").sum()) * wl.kv_bytes_per_token(w.num_kv_heads, w.head_dim)
    value = kv / dt / 1e9
    sample = ("%d of %d sequences (all %d heads, %d tokens) of the %s batch per step; fp64 C "
              "oracle on %d threads" % (len(ob.sample), w.num_seqs, w.num_heads,
                                        int(ob.lens.sum()), w.name, cores))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": args.gpus, "steps": steps, "warmup": warm, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": describe(w), "seed": w.seed, "sample": sample,
                   "parallelism": "replicas x%d" % max(args.gpus, 1)},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
