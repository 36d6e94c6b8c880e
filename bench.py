"""Paged decode benchmark: KV-read HBM GB/s (and % of peak) and seq-steps/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama70b|llama8b|heavytail|prefix] [--block-size BS]

One step = one decode step of the workload over all its layers: pa_copy_blocks of the
step's copy-on-write pairs (none unless the workload shares partial blocks), then per
layer the append of every sequence's newest token and decode over all cached tokens --
by default one pa_decode_append launch per layer (the append fused into decode; same
bits as the two calls), with --unfused pa_cache_append then pa_decode.  Inputs are
seeded synthetic tensors already resident in HBM; each layer's K/V pools (0.7 GB for
the default workload) are larger than L2, so no flush is needed.

With N > 1 (torchrun) every rank runs an independent replica of the workload (the
path has no exchange step); value = all ranks' KV bytes / the slowest rank's time.
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attn: KV-read HBM GB/s (% of B200 peak) and seq-steps/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0        # B200 HBM3e, nominal (the measured copy peak is the roofline)
L2_BYTES = 126 * 1024 * 1024


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest x over all ranks of the process group (x itself with one rank): the
    slowest rank's time is the job's time."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world: int, bytes_per_rank_step: int, ms_per_step: float) -> float:
    """Whole-job rate: every rank's bytes of one step over the (slowest rank's) step time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


def workload_desc(w, bs, layers=0, q_len=1):
    from paged_kv_cache_348_b200 import inputs

    ctx = {"tiny": "{5,16,17,40}", "llama8b": "U[128,2048]", "llama70b": "U[1000,8000]",
           "heavytail": "lognormal(median 512, sigma 1.2) clipped [16,32768]",
           "prefix": "2048 shared + U[0,512] private"}[w.name]
    return ("%s-shape paged decode step: %d layer(s), batch %d, %d q / %d kv heads, head_dim %d, "
            "block_size %d, %s, context lens %s, seed %d" % (
                w.name, layers or w.layers, w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, bs,
                w.dtype, ctx, w.seed)) + (", %d new tokens per sequence (causal)" % q_len
                                          if q_len > 1 else "")


def source_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "paged_kv_cache_348_b200", "csrc")
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(workload_name, bs, variant):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on
    the current kernel source for this workload, block size and entry point (variant:
    append, decode, e4m3, multi, cascade)."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d["entries"]["%s_bs%d_%s" % (workload_name, bs, variant)]
        if e.get("source_hash") != source_hash():
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id=None):
        self.proc = None
        self.bus_id = bus_id

    def __enter__(self):
        try:
            cmd = ["nvidia-smi", "--query-gpu=pci.bus_id," + self.FIELDS,
                   "--format=csv,noheader,nounits", "-lms", "200"]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            if self.bus_id and parts[0].lower()[-12:] != self.bus_id.lower()[-12:]:
                continue
            rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = [s for s in sm if s >= 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows)}


def device_bus_id(torch):
    try:
        p = torch.cuda.get_device_properties(torch.cuda.current_device())
        return "%08x:%02x:%02x.0" % (getattr(p, "pci_domain_id", 0), p.pci_bus_id, p.pci_device_id)
    except Exception:
        return None


# ------------------------------------------------------------------------------- oracle
def oracle_sample(w, bs, max_seconds=15.0, device_batch=None, nthreads=None):
    """Time the CPU oracle on whole sequences of layer 0 until ~max_seconds of work, on
    all host cores (or nthreads).  Returns (kv_bytes, seconds, seqs, threads)."""
    import torch

    import oracle
    from paged_kv_cache_348_b200 import inputs

    threads = nthreads or (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
                           else os.cpu_count())
    if device_batch is not None:
        b = device_batch
        def bits(t):
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.uint8:
                return t.numpy()
            return t.view(torch.int16).numpy().view(np.uint16)
        q, k, v = bits(b.q[0]), bits(b.k_caches[0]), bits(b.v_caches[0])
        tables, ctx = b.block_tables.cpu().numpy(), b.context_lens.cpu().numpy()
    else:
        q, k, v, tables, ctx = oracle_inputs(w, bs)
    order = list(range(len(ctx)))
    done_bytes, spent, seqs = 0, 0.0, 0
    chunk = max(1, threads // 8)
    i = 0
    while i < len(order) and spent < max_seconds:
        items = order[i:i + chunk]
        t0 = time.perf_counter()
        if k.dtype == np.uint8 and getattr(b, "kv_bscales", None) is not None:
            oracle.decode_e4m3_bs(q, k, v, b.kv_bscales[0][0].cpu().numpy(),
                                  b.kv_bscales[0][1].cpu().numpy(), tables, ctx,
                                  1.0 / math.sqrt(w.head_dim), w.dtype, items=items,
                                  nthreads=threads)
        elif k.dtype == np.uint8:
            oracle.decode_e4m3(q, k, v, *b.kv_scales, tables, ctx, 1.0 / math.sqrt(w.head_dim),
                               w.dtype, items=items, nthreads=threads)
        else:
            fn = oracle.decode if q.ndim == 3 else oracle.decode_multi
            fn(q, k, v, tables, ctx, 1.0 / math.sqrt(w.head_dim), w.dtype, items=items,
               nthreads=threads)
        spent += time.perf_counter() - t0
        done_bytes += int(sum(int(ctx[s]) for s in items)) * w.num_kv_heads * w.head_dim * 2 * \
            k.dtype.itemsize
        seqs += len(items)
        i += chunk
    return done_bytes, spent, seqs, threads


def oracle_inputs(w, bs):
    """Layer 0 of the workload for the oracle arm, built without the library: block tables
    from the oracle's reference block manager (the same seeded pool order and, for the
    shared-prefix workload, the same forks and appends as the GPU workload), values from
    the seeded generators with the streams the GPU workload uses."""
    import torch

    from oracle.cow import RefBlockManager
    from paged_kv_cache_348_b200 import inputs

    ctx = [int(c) for c in inputs.context_lens(w)]
    if w.name == "prefix":
        need = inputs.PREFIX_PROMPTS * (inputs.PREFIX_LEN // bs) + sum(
            -(-(c - inputs.PREFIX_LEN) // bs) for c in ctx)
    else:
        need = sum(-(-c // bs) for c in ctx)
    N = w.pool_blocks if w.pool_blocks else int(math.ceil(w.pool_factor * need))
    bm = RefBlockManager(N, bs, inputs.pool_order(N, w.seed))
    if w.name == "prefix":
        sids = []
        for p in range(inputs.PREFIX_PROMPTS):
            root = bm.new_seq(inputs.PREFIX_LEN)
            kids = [root] + [bm.fork(root) for _ in range(inputs.PREFIX_SAMPLES - 1)]
            for j, sid in enumerate(kids):
                for _ in range(ctx[p * inputs.PREFIX_SAMPLES + j] - inputs.PREFIX_LEN):
                    bm.append_slot(sid)
                sids.append(sid)
    else:
        sids = [bm.new_seq(c) for c in ctx]
    M = max(1, max(len(bm.tables[s]) for s in sids))
    tables = np.zeros((len(sids), M), dtype=np.int32)
    for i, s in enumerate(sids):
        tables[i, :len(bm.tables[s])] = bm.tables[s]
    lens = np.array([bm.ctx[s] for s in sids], dtype=np.int32)

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    shape = (N, w.num_kv_heads, bs, w.head_dim)
    k = bits(inputs.randn(shape, w.dtype, w.seed, "cpu", stream=1000))
    v = bits(inputs.randn(shape, w.dtype, w.seed, "cpu", stream=1001))
    q = bits(inputs.randn((len(sids), w.num_q_heads, w.head_dim), w.dtype, w.seed, "cpu",
                          stream=5000))
    return q, k, v, tables, lens


def run_reference(args, w, bs, rank, world):
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample(w, bs, max_seconds=1.0)
    t_all, b_all, s_all, threads = 0.0, 0, 0, 1
    per = max(5.0, 20.0 / max(1, args.steps))
    for _ in range(args.steps):
        nbytes, sec, seqs, threads = oracle_sample(w, bs, max_seconds=per)
        t_all += sec
        b_all += nbytes
        s_all += seqs
    gbs = b_all / t_all / 1e9
    # the metric's step is all layers of the workload: scale the sampled time
    layer_bytes = b_all / max(1, s_all)
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * (t_all / max(1, s_all)) * w.num_seqs * w.layers,
        "ms_per_step_extrapolated": True,
        "ms_per_step_basis": "oracle time per sampled whole sequence of layer 0, x %d sequences "
                             "x %d layers (the step is never run whole on the CPU)" % (
                                 w.num_seqs, w.layers),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload_desc(w, bs), "parallelism": "cpu"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": "%d whole sequences of layer 0 per step (%.1f s of oracle "
                                   "time per step), KV bytes of those sequences" % (
                                       s_all // max(1, args.steps), t_all / max(1, args.steps))},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "seq_steps_per_s": (s_all / w.layers) / t_all,
        "kv_bytes_per_seq_layer": layer_bytes,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------- ours
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=150)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama70b")
    ap.add_argument("--block-size", type=int, default=0)
    ap.add_argument("--unfused", action="store_true",
                    help="per layer pa_cache_append then pa_decode (default: pa_decode_append, "
                         "one launch, where the step has one new token per sequence)")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="8-bit E4M3 KV pools (pa_cache_append_e4m3 + pa_decode_e4m3)")
    ap.add_argument("--kv-fp8-block", action="store_true",
                    help="8-bit E4M3 KV pools with per-(block, kv head) scales "
                         "(pa_cache_append_e4m3_bs + pa_decode_e4m3_bs)")
    ap.add_argument("--cascade", action="store_true",
                    help="decode with pa_decode_cascade (shared prefixes read once per chunk)")
    ap.add_argument("--q-len", type=int, default=1,
                    help="new tokens per sequence (pa_decode_multi when > 1)")
    ap.add_argument("--layers", type=int, default=0,
                    help="layers of the workload to run (0: all; fewer only for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads' per-launch measurements")
    ap.add_argument("--secondary-iters", type=int, default=20)
    args = ap.parse_args()

    from paged_kv_cache_348_b200 import inputs

    w = inputs.WORKLOADS[args.workload]
    bs = args.block_size or w.block_size
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, w, bs, rank, world)

    import torch
    import torch.distributed as dist

    from paged_kv_cache_348_b200 import pagedkv as pk
    from paged_kv_cache_348_b200 import workload as wl

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    pk.load()
    if w.name == "prefix":
        b = wl.build_prefix_decode(w, device="cuda")
    else:
        b = wl.build(w, device="cuda", block_size=bs, layers=args.layers or None,
                     q_len=args.q_len, kv8="block" if args.kv_fp8_block else args.kv_fp8)
    if args.cascade:
        wl.use_cascade(b)
    stream = torch.cuda.current_stream()
    L = b.layers
    fused = not args.unfused and b.q_len == 1 and b.cascade is None and b.kv_scales is None
    kv_step = b.kv_bytes_per_step()
    kv_layer = kv_step // L

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        wl.run_step(b, fused=fused)
    barrier()
    if int(b.status.item()):
        raise RuntimeError("device status 0x%x after warm-up" % int(b.status.item()))

    # ---------------- timed region: K plain steps (no events between kernels, so
    # consecutive launches can overlap through programmatic dependent launch)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    launches = 0
    clocks = ClockSampler(device_bus_id(torch) if rank == 0 else None)
    with clocks:
        barrier()
        t_start.record(stream)
        for s in range(args.steps):
            wl.run_step(b, fused=fused)
            launches += L * (1 if fused else 2) * (2 if b.cascade is not None else 1) + \
                (1 if b.cow_pairs is not None and b.cow_pairs.shape[0] else 0)
        t_end.record(stream)
        barrier()
    ms = t_start.elapsed_time(t_end)
    ms_local = ms
    # ---------------- roofline region: the same steps with an event pair around every
    # pa_decode launch, for that kernel's own average duration (the events serialise the
    # launches; when every launch of the timed region above is the decode kernel, that
    # region's time per launch is used instead, and this one is reported beside it)
    rsteps = max(1, min(args.steps, 20))
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(rsteps * L)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(rsteps * L)]
    barrier()
    for s in range(rsteps):
        if b.cow_pairs is not None and b.cow_pairs.shape[0]:
            pk.pa_copy_blocks(b.k_caches, b.v_caches, b.cow_pairs, b.status)
        for l in range(L):
            if fused:
                pass
            elif b.kv_bscales is not None:
                pk.pa_cache_append_e4m3_bs(b.k_caches[l], b.v_caches[l], *b.kv_bscales[l],
                                           b.k_new[l], b.v_new[l], b.slot_mapping, b.status)
            elif b.kv_scales is not None:
                pk.pa_cache_append_e4m3(b.k_caches[l], b.v_caches[l], b.k_new[l], b.v_new[l],
                                        b.slot_mapping, *b.kv_scales, b.status)
            else:
                pk.pa_cache_append(b.k_caches[l], b.v_caches[l], b.k_new[l], b.v_new[l],
                                   b.slot_mapping, b.status)
            ev_s[s * L + l].record(stream)
            if fused:
                wl.append_decode_layer(b, l)
            else:
                wl.decode_layer(b, l)
            ev_e[s * L + l].record(stream)
    barrier()
    dec_ms = [a.elapsed_time(e) for a, e in zip(ev_s, ev_e)]
    ms = max_over_ranks(ms, world)
    st = int(b.status.item())
    if st:
        raise RuntimeError("device status 0x%x in the timed region" % st)
    ms_step = ms / args.steps
    value = job_gbs(world, kv_step, ms_step)
    peak, peak_kind = measured_hbm_peak()
    dec_avg_events = statistics.mean(dec_ms)
    dec_med_events = statistics.median(dec_ms)
    only_decode = fused and not (b.cow_pairs is not None and b.cow_pairs.shape[0])
    if only_decode:
        dec_avg = ms_local / (args.steps * L)
        dec_src = "timed region / launches (every launch in the timed region is this kernel)"
    else:
        dec_avg = dec_avg_events
        dec_src = "an event pair around each launch"
    achieved = kv_layer / (dec_avg * 1e-3) / 1e9
    variant = ("cascade" if b.cascade is not None else
               "e4m3bs_append" if fused and b.kv_bscales is not None else
               "append" if fused else
               "e4m3bs" if b.kv_bscales is not None else
               "e4m3" if b.kv_scales is not None else "decode" if b.q_len == 1 else "multi")
    traffic = ncu_traffic(w.name, bs, variant)

    # ---------------- end to end through the public API, host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(b, args, world, kv_step, fused)

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype + ("+e4m3 kv, per-(block, kv head) scales" if b.kv_bscales is not None
                            else "+e4m3 kv" if b.kv_scales is not None else ""),
        "data": "synthetic",
        "config": {"workload": workload_desc(w, bs, b.layers, b.q_len), "global_batch": w.num_seqs * world,
                   "seq_len": float(b.context_lens.float().mean().item()),
                   "parallelism": "replicas" if world > 1 else "single gpu",
                   "l2": "inputs larger than L2 (%.2f GB of K/V per layer)" % (kv_layer / 1e9)},
        "pct_of_peak_hbm": 100.0 * value / world / peak,
        "peak_hbm_gbs": peak, "peak_kind": peak_kind,
        "pct_of_nominal_hbm": 100.0 * value / world / NOMINAL_HBM_GBS,
        "nominal_hbm_gbs": NOMINAL_HBM_GBS,
        "seq_steps_per_s": world * w.num_seqs / (ms_step * 1e-3),
        "kv_bytes_per_step": kv_step,
        "roofline": {"bound": "hbm", "kernel": "pa_decode_split_kernel (%s)" % (
                         "two launches per pa_decode_cascade" if b.cascade is not None else
                         "one launch per pa_decode_append_e4m3_bs" if fused and
                         b.kv_bscales is not None else
                         "one launch per pa_decode_append" if fused else
                         "one launch per pa_decode_e4m3_bs" if b.kv_bscales is not None else
                         "one launch per pa_decode_e4m3" if b.kv_scales is not None else
                         "one launch per pa_decode" if b.q_len == 1 else
                         "one launch per pa_decode_multi"),
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": kv_layer,
                     "avg_launch_ms": dec_avg, "avg_launch_ms_from": dec_src,
                     "avg_launch_ms_event_pairs": dec_avg_events,
                     "median_launch_ms_event_pairs": dec_med_events,
                     "launches_timed": args.steps * L if only_decode else len(dec_ms),
                     "peak_source": peak_kind},
        "gpu_launches": launches,
        "clocks": clocks.summary() if rank == 0 else None,
        "e2e": e2e,
    }
    if w.name == "prefix":
        # shared blocks counted once: the bytes a read-once-per-block schedule needs
        uniq = b.unique_kv_bytes_per_step()
        line["kv_bytes_unique_per_step"] = uniq
        line["roofline_unique_bytes"] = {
            "achieved": uniq / L / (dec_avg * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
            "frac": uniq / L / (dec_avg * 1e-3) / 1e9 / peak}
    if w.name == "llama70b" and not args.no_secondary and b.q_len == 1 and b.kv_scales is None \
            and b.cascade is None:
        # the other workloads, built one at a time beside the step's buffers
        line["secondary"] = secondary_measurements(args, peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nbytes, sec, seqs, threads = oracle_sample(w, bs, device_batch=b)
        n1, sec1, seqs1, _ = oracle_sample(w, bs, max_seconds=3.0, device_batch=b, nthreads=1)
        line["cpu_baseline"] = {
            "value": nbytes / sec / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": "%d whole sequences (all %d q heads) of layer 0 of this workload, "
                      "%.1f s" % (seqs, w.num_q_heads, sec),
            "value_1thread": n1 / sec1 / 1e9,
            "sample_1thread": "%d whole sequences of layer 0, %.1f s on one thread" % (seqs1, sec1)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(b, args, world, kv_step, fused=False):
    """The step through the public API with host buffers.  Every step copies, from pinned
    host memory, every layer's new q / k / v, the block tables, context lens and slot
    mapping, runs append + decode per layer, and copies every layer's output back.
    Copies run on their own streams and the device buffers of a step are double-buffered
    across steps: step i+1's inputs upload while step i computes, and step i's outputs
    are read back while step i+1 computes; the compute stream waits twice per step (its
    inputs are in, the read-back of the outputs it overwrites is done), so the layers'
    launches follow each other directly.  Timed with CUDA events from the first upload to
    the last read-back."""
    import torch

    from paged_kv_cache_348_b200 import pagedkv as pk
    from paged_kv_cache_348_b200 import workload as wl

    L = b.layers
    hq = [t.cpu().pin_memory() for t in b.q]
    hk = [t.cpu().pin_memory() for t in b.k_new]
    hv = [t.cpu().pin_memory() for t in b.v_new]
    hctx = b.context_lens.cpu().pin_memory()
    htab = b.block_tables.cpu().pin_memory()
    hslot = b.slot_mapping.cpu().pin_memory()
    hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in b.out]
    h2d_bytes = sum(t.numel() * t.element_size() for t in hq + hk + hv + [hctx, htab, hslot])
    d2h_bytes = sum(t.numel() * t.element_size() for t in hout)
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    # two sets of a step's device buffers (set m serves the steps i with i % 2 == m)
    own = (b.q, b.k_new, b.v_new, b.out, b.block_tables, b.context_lens, b.slot_mapping)
    qs = [b.q, [t.clone() for t in b.q]]
    ks = [b.k_new, [t.clone() for t in b.k_new]]
    vs = [b.v_new, [t.clone() for t in b.v_new]]
    outs = [b.out, [t.clone() for t in b.out]]
    tabs = [b.block_tables, b.block_tables.clone()]
    ctxs = [b.context_lens, b.context_lens.clone()]
    slots = [b.slot_mapping, b.slot_mapping.clone()]
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]     # set m's inputs are on the device
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]   # set m's step computed
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]    # set m's outputs are on the host

    def step(i):
        m = i % 2
        with torch.cuda.stream(up):
            up.wait_event(ev_used[m])                    # step i-2 is done with set m
            tabs[m].copy_(htab, non_blocking=True)
            ctxs[m].copy_(hctx, non_blocking=True)
            slots[m].copy_(hslot, non_blocking=True)
            for l in range(L):
                qs[m][l].copy_(hq[l], non_blocking=True)
                ks[m][l].copy_(hk[l], non_blocking=True)
                vs[m][l].copy_(hv[l], non_blocking=True)
            ev_in[m].record(up)
        comp.wait_event(ev_in[m])
        comp.wait_event(ev_out[m])                       # step i-2's outputs are read back
        b.q, b.k_new, b.v_new, b.out = qs[m], ks[m], vs[m], outs[m]
        b.block_tables, b.context_lens, b.slot_mapping = tabs[m], ctxs[m], slots[m]
        if fused:
            wl.run_step(b, comp, fused=True)
        else:
            for l in range(L):
                if b.kv_bscales is not None:
                    pk.pa_cache_append_e4m3_bs(b.k_caches[l], b.v_caches[l], *b.kv_bscales[l],
                                               b.k_new[l], b.v_new[l], b.slot_mapping, b.status,
                                               comp)
                elif b.kv_scales is not None:
                    pk.pa_cache_append_e4m3(b.k_caches[l], b.v_caches[l], b.k_new[l],
                                            b.v_new[l], b.slot_mapping, *b.kv_scales, b.status,
                                            comp)
                else:
                    pk.pa_cache_append(b.k_caches[l], b.v_caches[l], b.k_new[l], b.v_new[l],
                                       b.slot_mapping, b.status, comp)
                wl.decode_layer(b, l, comp)
        ev_used[m].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev_used[m])
            for l in range(L):
                hout[l].copy_(outs[m][l], non_blocking=True)
            ev_out[m].record(down)

    try:
        for i in range(max(1, args.warmup)):
            step(i)
        torch.cuda.synchronize()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(comp)
        up.wait_event(s)
        down.wait_event(s)
        for i in range(args.steps):
            step(i)
        comp.wait_event(ev_out[(args.steps - 1) % 2])
        e.record(comp)
        torch.cuda.synchronize()
    finally:
        b.q, b.k_new, b.v_new, b.out, b.block_tables, b.context_lens, b.slot_mapping = own
    ms = max_over_ranks(s.elapsed_time(e), world)
    ms_step = ms / args.steps
    return {"value": job_gbs(world, kv_step, ms_step), "unit": "GB/s",
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
            "ms_per_step": ms_step,
            "copies": "pinned host buffers; uploads and read-backs on two copy streams, "
                      "device buffers double-buffered across steps (each step's copies "
                      "overlap the neighbouring steps' compute)"}



# ------------------------------------------------------------------------------- secondary
def time_launches(torch, fn, n, warmup, flush=None):
    """Device time of fn() (one decode call: one or two library launches on the current
    stream) with an event pair around each call; `flush` (an L2 flush) runs before each
    timed call, outside the events.  Returns (median ms, mean ms)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = []
    for _ in range(n):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        e.record()
        evs.append((a, e))
    torch.cuda.synchronize()
    ts = [a.elapsed_time(e) for a, e in evs]
    return statistics.median(ts), statistics.mean(ts)


def tail_waste_table():
    """Fraction of held cache slots that hold no token (the unused tail of each
    sequence's last block; shared blocks counted once per sequence), per workload and
    block size: host bookkeeping only."""
    from paged_kv_cache_348_b200 import inputs
    from paged_kv_cache_348_b200.block_manager import BlockManager

    out = {}
    for name in ("tiny", "llama8b", "llama70b", "prefix", "heavytail"):
        w = inputs.WORKLOADS[name]
        ctx = [int(c) for c in inputs.context_lens(w)]
        row = {}
        for bs in (1, 8, 16, 32):
            held = sum(-(-c // bs) * bs for c in ctx)
            row["bs%d" % bs] = (held - sum(ctx)) / held
        if name == "prefix":
            # the shared 2048-token prefix is held once per prompt (block aligned at
            # these sizes), the private tokens per sample
            for bs in (1, 8, 16, 32):
                bm = BlockManager(10 ** 6, bs)
                sids = []
                for p in range(inputs.PREFIX_PROMPTS):
                    root = bm.allocate(inputs.PREFIX_LEN)
                    kids = [root] + [bm.fork(root) for _ in range(inputs.PREFIX_SAMPLES - 1)]
                    for j, sid in enumerate(kids):
                        for _ in range(ctx[p * inputs.PREFIX_SAMPLES + j] - inputs.PREFIX_LEN):
                            bm.append_token(sid)
                        sids.append(sid)
                held_slots = (10 ** 6 - bm.free_blocks) * bs
                row["bs%d_unique" % bs] = (held_slots - (inputs.PREFIX_PROMPTS * inputs.PREFIX_LEN +
                                                         sum(c - inputs.PREFIX_LEN for c in ctx))) \
                    / held_slots
        out[name] = row
    return out


def secondary_measurements(args, peak):
    """Per-launch device time, KV-read rate and roofline fraction of the other workloads
    (each built on its own, measured, and freed): the 8B shape, the heavy-tailed batch at
    every block size, the shared-prefix batch (plain and cascade), 8-bit pools, several
    new tokens per sequence, and identity (contiguous) against fragmented placement.  Calls
    are timed one at a time with an event pair; when a layer's K/V pools are under 4x the
    L2 size, a 256 MB buffer is written before each timed call so the pools come from
    HBM."""
    import torch

    from paged_kv_cache_348_b200 import inputs
    from paged_kv_cache_348_b200 import workload as wl

    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = {}

    def measure(name, b, fn, note, kv_bytes=None, unique=None, launches=1):
        pool = 2 * b.k_caches[0].numel() * b.k_caches[0].element_size()
        flush = pool < 4 * L2_BYTES
        med, mean = time_launches(torch, fn, args.secondary_iters, 3,
                                  (lambda: flush_buf.zero_()) if flush else None)
        st = int(b.status.item())
        if st:
            raise RuntimeError("%s: device status 0x%x" % (name, st))
        kvb = kv_bytes if kv_bytes is not None else b.kv_bytes_per_step() // b.layers
        e = {"workload": note, "median_ms": med, "mean_ms": mean, "kv_bytes": kvb,
             "gbs": kvb / (med * 1e-3) / 1e9, "frac": kvb / (med * 1e-3) / 1e9 / peak,
             "launches_per_call": launches, "l2_flush": flush,
             "seqs_per_s": len(b.sids) / (med * 1e-3)}
        if unique is not None:
            e["unique_kv_bytes"] = unique
            e["unique_gbs"] = unique / (med * 1e-3) / 1e9
            e["unique_frac"] = e["unique_gbs"] / peak
        out[name] = e

    def fused(b):
        return lambda: wl.append_decode_layer(b, 0)

    def plain(b):
        return lambda: wl.decode_layer(b, 0)

    runs = [
        ("llama70b_layer", lambda: wl.build(inputs.LLAMA70B, layers=1), fused,
         "70B shape, one layer, fragmented placement, pa_decode_append"),
        ("llama70b_layer_identity", lambda: wl.build(inputs.LLAMA70B, layers=1, contiguous=True),
         fused, "70B shape, one layer, identity (contiguous) placement, pa_decode_append"),
        ("llama70b_q2", lambda: wl.build(inputs.LLAMA70B, layers=1, q_len=2), plain,
         "70B shape, 2 new tokens a sequence (16 query rows per kv head), pa_decode_multi"),
        ("llama70b_q4", lambda: wl.build(inputs.LLAMA70B, layers=1, q_len=4), plain,
         "70B shape, 4 new tokens (32 rows), pa_decode_multi"),
        ("llama70b_q8", lambda: wl.build(inputs.LLAMA70B, layers=1, q_len=8), plain,
         "70B shape, 8 new tokens (64 rows), pa_decode_multi"),
        ("llama70b_e4m3", lambda: wl.build(inputs.LLAMA70B, layers=1, kv8=True), plain,
         "70B shape, one layer, 8-bit E4M3 pools (bytes counted at 1 per value), "
         "pa_decode_e4m3"),
        ("llama70b_e4m3_bs", lambda: wl.build(inputs.LLAMA70B, layers=1, kv8="block"), plain,
         "70B shape, one layer, 8-bit E4M3 pools with per-(block, kv head) scales, "
         "pa_decode_e4m3_bs"),
        ("llama70b_e4m3_bs_append", lambda: wl.build(inputs.LLAMA70B, layers=1, kv8="block"),
         fused, "70B shape, one layer, 8-bit E4M3 pools with per-(block, kv head) scales, "
         "pa_decode_append_e4m3_bs (the newest token quantised and appended in the launch)"),
        ("llama8b", lambda: wl.build(inputs.LLAMA8B), fused, "8B shape, pa_decode_append"),
        ("llama8b_q4", lambda: wl.build(inputs.LLAMA8B, q_len=4), plain,
         "8B shape, 4 new tokens (16 rows), pa_decode_multi"),
        ("llama8b_e4m3", lambda: wl.build(inputs.LLAMA8B, kv8=True), plain,
         "8B shape, 8-bit E4M3 pools, pa_decode_e4m3"),
    ]
    for bs in (1, 8, 16, 32):
        runs.append(("heavytail_bs%d" % bs,
                     (lambda bs=bs: wl.build(inputs.HEAVYTAIL, block_size=bs)), fused,
                     "heavy-tailed 256 sequences, block_size %d, pa_decode_append" % bs))
    runs.append(("heavytail_bs16_identity",
                 lambda: wl.build(inputs.HEAVYTAIL, block_size=16, contiguous=True), fused,
                 "heavy-tailed, block_size 16, identity (contiguous) placement"))
    runs.append(("heavytail_bs16_e4m3_bs",
                 lambda: wl.build(inputs.HEAVYTAIL, block_size=16, kv8="block"), plain,
                 "heavy-tailed, block_size 16, 8-bit pools with per-(block, kv head) scales"))
    runs.append(("heavytail_bs1_e4m3",
                 lambda: wl.build(inputs.HEAVYTAIL, block_size=1, kv8=True), plain,
                 "heavy-tailed, block_size 1, 8-bit E4M3 pools"))
    for name, mk, how, note in runs:
        b = mk()
        measure(name, b, how(b), note)
        del b
        torch.cuda.empty_cache()
    b = wl.build_prefix_decode()
    uniq = b.unique_kv_bytes_per_step()
    measure("prefix_plain", b, plain(b), "shared prefix (16 prompts x 8 samples), pa_decode; "
            "gbs on logical bytes (a shared block once per reader)", unique=uniq)
    wl.use_cascade(b)
    measure("prefix_cascade", b, plain(b), "shared prefix, pa_decode_cascade (prefix pass + "
            "suffix pass)", unique=uniq, launches=2)
    del b
    torch.cuda.empty_cache()
    out["tail_waste"] = tail_waste_table()
    return out

if __name__ == "__main__":
    sys.exit(main())
