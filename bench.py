"""Benchmark of the SegmentAttention hot path on B200.

One step = one pass of the whole path over one batch of the long-context mix
(8 decode requests at k = 131072, then one prefill chunk of 2048 queries over
131072 prior tokens; 64 query / 8 kv heads, d = 128, shared segmented pool):
table build is done once (host), then per step: decode split-K + merge and
the tcgen05 prefill, all through the C ABI on one stream.

Metric: prefill TFLOPS and decode HBM GB/s vs peak, as in the Flood README
kernel table ("Kernels > Seg-attn", which reports both prefill and decode in
TFLOPS).  `value` is the step's attention TFLOP/s: (prefill flops, causal
4*d*Hq*sum(q*p + q^2/2), plus decode flops 4*d*Hq*sum(k)) / step time.  The
per-leg numbers (prefill TFLOP/s, decode GB/s) and their fractions of the
measured peaks are in `legs`.

The default run (config 5, one GPU) adds `configs`: one record each for the
pages' q = k = 1024 prefill (config 2), the chunked varlen prefill (config 3)
and the batched decode (config 4), timed call by call with L2 flushed before
each call, with their fractions of the measured peaks and an oracle parity
sample.

Configs 6 and 7 are the shared-prefix workloads (prefix caching): their tables
are built with SEG_ATTN_SHARE_PREFIX, and the same step without sharing is timed
beside them (`legs.*.plain_ms`).  Their decode roofline counts each distinct K/V
slot once (the bytes a shared-prefix job must move).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import segmented_kv_cache_b200 as sa  # noqa: E402
from segmented_kv_cache_b200 import synth  # noqa: E402

METRIC = "prefill TFLOPS and decode HBM GB/s (1 B200) vs peak; max-abs err vs oracle"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def prefill_flops(batch, wl):
    tot = 0.0
    for q, k in zip(batch.q_lens, batch.k_lens):
        p = k - q
        tot += q * p + (q * q / 2.0 if batch.causal else q * q)
    return 4.0 * wl.head_dim * wl.q_heads * tot


def decode_flops(batch, wl):
    return 4.0 * wl.head_dim * wl.q_heads * float(sum(batch.k_lens))


def decode_bytes(batch, wl, table_bytes, kv_bytes=2):
    kv = 2 * kv_bytes * wl.kv_heads * wl.head_dim * float(sum(batch.k_lens))
    qo = 2 * 2 * batch.batch * wl.q_heads * wl.head_dim
    return kv + qo + 4 * batch.batch * wl.q_heads + table_bytes


def distinct_slots(batch):
    """Number of distinct pool slots the batch's segment lists name."""
    runs = sorted((s, s + l) for ss, ll in zip(batch.seg_starts, batch.seg_lens)
                  for s, l in zip(ss, ll) if l > 0)
    n, end = 0, -1
    for a, b in runs:
        if b > end:
            n += b - max(a, end)
            end = b
    return n


def decode_bytes_distinct(batch, wl, table_bytes, kv_bytes=2):
    """decode_bytes with every distinct K/V slot counted once (shared prefixes)."""
    kv = 2 * kv_bytes * wl.kv_heads * wl.head_dim * float(distinct_slots(batch))
    qo = 2 * 2 * batch.batch * wl.q_heads * wl.head_dim
    return kv + qo + 4 * batch.batch * wl.q_heads + table_bytes


def launches_of(desc):
    """Kernel launches one compute call makes for a built table."""
    shared = desc.shared == 1
    n = 0
    if shared and desc.num_group_work > 0:  # pass over the shared prefixes (two-tile, one-tile)
        n += (desc.num_group_work > desc.num_group_single) + (desc.num_group_single > 0)
    if desc.mode == sa.MODE_PREFILL:
        n += (desc.num_work > desc.num_single) + (desc.num_single > 0)
        n += 1 if desc.num_merge > 0 else 0
    else:
        n += 1 if desc.num_work > 0 else 0
        n += 1 if (desc.workspace_bytes > 0 and not shared) else 0
    if shared and desc.num_cascade > 0:
        n += 1
    return n


def _local_includes(path, seen):
    """`path` and every header of the repo it includes (quoted #include, recursively)."""
    if path in seen:
        return
    seen.append(path)
    here = os.path.dirname(path)
    with open(path, "r", errors="replace") as f:
        names = re.findall(r'^\s*#\s*include\s*"([^"]+)"', f.read(), flags=re.M)
    for name in names:
        for d in (here, os.path.join(ROOT, "include")):
            cand = os.path.normpath(os.path.join(d, name))
            if os.path.exists(cand):
                _local_includes(cand, seen)
                break


def source_digest(path):
    """sha256[:16] over a kernel source and the repo headers it includes, so a change to a
    shared header (barrier waits, table layout) also marks old counters as stale."""
    files = []
    _local_includes(os.path.abspath(path), files)
    h = hashlib.sha256()
    for fp in [files[0]] + sorted(files[1:]):
        with open(fp, "rb") as f:
            h.update(os.path.basename(fp).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload_tag):
    """DRAM bytes per launch from the committed ncu summary, if it still matches the source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload_tag}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"dram bytes per launch \(read\+write\):\s*([0-9.eE+]+)", text)
    h = re.search(r"source sha256\[:16\] of ([\w/.]+) with its headers:\s*([0-9a-f]{16})", text)
    if not m or not h:
        return None
    src = os.path.join(ROOT, h.group(1))
    if not os.path.exists(src) or source_digest(src) != h.group(2):
        return None  # kernel changed since the counters were taken
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [l for (t, l) in self.lines if t0 - 0.06 <= t <= t1 + 0.06] or \
            [l for (_, l) in self.lines[-3:]]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 10:
                continue
            try:
                sm.append(float(f[2]))
                mx.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def rank_seed(config, rank):
    """Weak scaling: every rank draws its own batch of the same shape."""
    return config - 1 + 1000 * rank


def max_over_ranks(value, dist=None, device="cpu"):
    """Max of a per-rank timing over all ranks (the job ends with the slowest rank)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank_step, ms_total, steps):
    """Whole-job rate: units processed by all ranks / the slowest rank's time."""
    return world * units_per_rank_step / (ms_total * 1e-3 / steps)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- workload
class Path:
    """Device-resident buffers + tables of one workload, and the calls of one step."""

    def __init__(self, wl, device, kv_dtype="bf16", share=False):
        self.wl = wl
        self.device = device
        self.legs = []
        self.kv_dtype = kv_dtype
        if kv_dtype == "fp8":  # every leg reads E4M3 copies of the pools
            self.k8, self.v8, self.ks, self.vs = synth.fp8_pools(wl.k_pool, wl.v_pool)
        for b in wl.batches:
            mode = sa.MODE_PREFILL if b.mode == "prefill" else sa.MODE_DECODE
            tab = sa.SegTable.build(b.q_lens if mode == sa.MODE_PREFILL else None, b.seg_starts,
                                    b.seg_lens, wl.num_slots, b.causal,
                                    mode | (sa.SHARE_PREFIX if share else 0), wl.q_heads,
                                    wl.kv_heads, wl.head_dim, pin=True)
            tab.to(device)
            out = torch.empty_like(b.q)
            lse = torch.empty(b.q.shape[0], wl.q_heads, dtype=torch.float32, device=device)
            ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device=device)
                  if tab.workspace_bytes else None)
            launches = launches_of(tab.desc)
            self.legs.append(dict(batch=b, mode=mode, tab=tab, out=out, lse=lse, ws=ws,
                                  launches=launches))

    def run_leg(self, leg, stream=None):
        if self.kv_dtype == "fp8":
            fn = (sa.seg_attn_prefill_fp8 if leg["mode"] == sa.MODE_PREFILL
                  else sa.seg_attn_decode_fp8)
            fn(leg["batch"].q, self.k8, self.v8, self.ks, self.vs, leg["out"], leg["lse"],
               leg["tab"].device, leg["tab"].desc, self.wl.scale, leg["ws"], stream)
            return
        fn = sa.seg_attn_prefill if leg["mode"] == sa.MODE_PREFILL else sa.seg_attn_decode
        fn(leg["batch"].q, self.wl.k_pool, self.wl.v_pool, leg["out"], leg["lse"],
           leg["tab"].device, leg["tab"].desc, self.wl.scale, leg["ws"], stream)

    def launches_per_step(self):
        return sum(l["launches"] for l in self.legs)


def workload_name(wl):
    return {1: "tiny causal prefill", 2: "pages-shaped prefill q=k=1024",
            3: "chunked prefill varlen (16 req, 2048 new tokens)",
            4: "batched decode 128 req k=1024..32768",
            5: "long-context mix: decode 8x131072 + prefill 2048 over 131072",
            6: "shared-prefix decode: 8 groups x 8 req, prefix 8192..32768 + own 512..4096",
            7: "shared-prefix chunked prefill: 4 groups x 8 req, prefix 4096..16384, "
               "chunks 4..32"}[wl.config]


# ----------------------------------------------------------------------------- oracle legs
def oracle_sample(wl, leg_batches, budget_rows, rng_seed=0):
    """Bounded oracle sample: `budget_rows` (token, head) rows per batch of the workload.

    Returns (flops, seconds, rows_desc, results) where results hold the oracle rows for a
    parity spot check of the GPU outputs."""
    import oracle
    g = torch.Generator().manual_seed(rng_seed)
    flops, secs, results, desc = 0.0, 0.0, [], []
    for bi, b in enumerate(leg_batches):
        n = min(budget_rows[bi], b.total_q * wl.q_heads)
        toks = torch.randint(0, b.total_q, (n,), generator=g)
        heads = torch.randint(0, wl.q_heads, (n,), generator=g)
        q_off = np.concatenate([[0], np.cumsum(b.q_lens)])
        reqs = sorted(set(int(np.searchsorted(q_off, int(t), side="right") - 1) for t in toks))
        # compact pool: only the sampled requests' segments (relocation is result-neutral)
        seg_s, seg_l, idx, pos = [], [], [], 0
        for r in reqs:
            ss, ll = [], []
            for s, l in zip(b.seg_starts[r], b.seg_lens[r]):
                ss.append(pos)
                ll.append(l)
                idx.append(torch.arange(s, s + l))
                pos += l
            seg_s.append(ss)
            seg_l.append(ll)
        ii = torch.cat(idx).to(wl.k_pool.device)
        kp, vp = wl.k_pool[ii].cpu(), wl.v_pool[ii].cpu()
        q_rows = torch.cat([torch.arange(q_off[r], q_off[r + 1]) for r in reqs])
        qc = b.q[q_rows.to(b.q.device)].cpu()
        new_off = np.concatenate([[0], np.cumsum([b.q_lens[r] for r in reqs])])
        remap = {}
        for j, r in enumerate(reqs):
            for t in range(b.q_lens[r]):
                remap[q_off[r] + t] = new_off[j] + t
        ltok = np.array([remap[int(t)] for t in toks], dtype=np.int64)
        for t in toks.tolist():
            r = int(np.searchsorted(q_off, t, side="right") - 1)
            i = t - q_off[r]
            vis = (b.k_lens[r] - b.q_lens[r] + i + 1) if (b.causal and b.mode == "prefill") else \
                b.k_lens[r]
            flops += 4.0 * wl.head_dim * min(vis, b.k_lens[r])
        t0 = time.perf_counter()
        o, l = oracle.attention([b.q_lens[r] for r in reqs], seg_s, seg_l, qc, kp, vp, wl.scale,
                                b.causal and b.mode == "prefill", rows=(ltok, heads.numpy()))
        secs += time.perf_counter() - t0
        results.append((bi, toks, heads, o, l))
        desc.append(f"{n} random (token, head) rows of the {b.mode} batch")
    return flops, secs, "; ".join(desc), results


# ----------------------------------------------------------------------------- main arms
def arm_config(wl, args, world, share):
    """The `config` object of the JSON line, the same for both arms."""
    pool_bytes = 2 * wl.k_pool.numel() * 2
    return {"workload": workload_name(wl) + ("" if args.context_scale == 1.0 else
                                             f" (context x{args.context_scale})"),
            "seed": wl.config - 1,
            "q_heads": wl.q_heads, "kv_heads": wl.kv_heads, "head_dim": wl.head_dim,
            "num_slots": wl.num_slots,
            "l2": ("inputs larger than L2 (pools %.1f GB), no flush" % (pool_bytes / 1e9))
            if pool_bytes > L2_BYTES else "inputs fit in L2",
            "parallelism": f"dp{world} (independent batches per GPU)",
            "share_prefix": bool(share), "kv_cache": args.kv_dtype}


def run_reference(args):
    """The oracle as it stands, timed on the host cores, on bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.make_workload(args.config, device="cuda" if torch.cuda.is_available() else "cpu",
                             context_scale=args.context_scale)
    rows = [args.ref_rows] * len(wl.batches)
    for _ in range(args.warmup if args.warmup <= 1 else 1):
        oracle_sample(wl, wl.batches, [max(1, r // 8) for r in rows], rng_seed=99)
    fl, sec = 0.0, 0.0
    sample_desc = ""
    for s in range(args.steps):
        f, t, sample_desc, _ = oracle_sample(wl, wl.batches, rows, rng_seed=s)
        fl += f
        sec += t
    value = fl / sec / 1e12
    cores = cpu_cores()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(wl, args, int(os.environ.get("WORLD_SIZE", "1")),
                                 args.share_prefix if args.share_prefix is not None
                                 else wl.config in (6, 7)),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step: {sample_desc}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    # weak scaling: every rank runs its own batch of the same shape (seed offset by rank)
    wl = synth.make_workload(args.config, device=str(device), seed=rank_seed(args.config, rank),
                             context_scale=args.context_scale)
    share = args.share_prefix if args.share_prefix is not None else wl.config in (6, 7)
    path = Path(wl, device, args.kv_dtype, share)
    stream = torch.cuda.current_stream(device)

    def step():
        for leg in path.legs:
            path.run_leg(leg)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert sa.seg_attn_take_device_error() == 0

    # per-leg events inside the timed region, on the launching (current) stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(path.legs) + 1)]
          for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local).start() if rank == 0 else None
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        for i, leg in enumerate(path.legs):
            path.run_leg(leg)
            ev[s][i + 1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if dist:
        dist.barrier()
    clocks = sampler.stop(t0, t1) if sampler else None
    ms = start.elapsed_time(end)
    leg_ms = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps)) / args.steps
              for i in range(len(path.legs))]
    ms = max_over_ranks(ms, dist, device)
    assert sa.seg_attn_take_device_error() == 0
    plain_ms = time_plain_legs(wl, device, args) if share else None

    peaks, peak_kind = load_peaks()
    flops_step = 0.0
    legs = {}
    dominant = None
    for leg, lm in zip(path.legs, leg_ms):
        b = leg["batch"]
        if leg["mode"] == sa.MODE_PREFILL:
            f = prefill_flops(b, wl)
            tf = f / (lm * 1e-3) / 1e12
            legs["prefill"] = {"ms": lm, "tflops": tf, "flops": f,
                               "frac_sustained": tf / peaks["bf16_tflops_sustained"],
                               "frac_burst": tf / peaks["bf16_tflops"],
                               "launches": leg["launches"]}
            flops_step += f
            cand = ("tensor", lm, f)
        else:
            f = decode_flops(b, wl)
            kvb = 1 if args.kv_dtype == "fp8" else 2
            by = decode_bytes(b, wl, leg["tab"].desc.table_bytes, kvb)
            if share:  # shared prefixes: the job must move each distinct slot once
                eff = by / (lm * 1e-3) / 1e9
                by = decode_bytes_distinct(b, wl, leg["tab"].desc.table_bytes, kvb)
            gbs = by / (lm * 1e-3) / 1e9
            legs["decode"] = {"ms": lm, "gbs": gbs, "bytes": by, "tflops": f / (lm * 1e-3) / 1e12,
                              "frac_hbm": gbs / peaks["hbm_gbs"],
                              "launches": leg["launches"]}
            if share:
                legs["decode"]["gbs_effective"] = eff  # every request's keys counted
            flops_step += f
            cand = ("hbm", lm, by)
        if dominant is None or cand[1] > dominant[1]:
            dominant = cand
    value = job_throughput(world, flops_step, ms, args.steps) / 1e12
    if plain_ms is not None:
        for leg, pm in zip(path.legs, plain_ms):
            name = "prefill" if leg["mode"] == sa.MODE_PREFILL else "decode"
            legs[name]["plain_ms"] = pm
            legs[name]["speedup_vs_plain"] = pm / legs[name]["ms"]
            legs[name]["shared_groups"] = int(leg["tab"].desc.num_groups)

    if dominant[0] == "tensor":
        achieved = dominant[2] / (dominant[1] * 1e-3) / 1e12
        # the prefill runs for milliseconds inside a timed region well under a second: the
        # burst cuBLAS figure is its peak; the power-capped sustained one is reported beside it
        peak = peaks["bf16_tflops"]
        fp8 = args.kv_dtype == "fp8"
        traffic = profiled_traffic("prefill_fp8_sm100" if fp8 else "prefill_sm100",
                                   f"cfg{wl.config}")
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "frac_sustained": achieved / peaks["bf16_tflops_sustained"],
                "kernel": "prefill_kernel<128> (E4M3 cache)" if fp8 else "prefill_kernel<128>",
                "peak_kind": f"{peak_kind} burst bf16 (cuBLAS 8192^3, best of 10)"}
    else:
        achieved = dominant[2] / (dominant[1] * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        traffic = profiled_traffic("decode_sm100", f"cfg{wl.config}")
        kern = ("prefill_kernel<128> over shared prefixes + decode_chunk_kernel<128> + "
                "cascade_merge_kernel<128>" if share else
                "decode_chunk_kernel<128> + decode_merge_kernel<128>")
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "kernel": kern,
                "peak_kind": f"{peak_kind} copy bandwidth"}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if args.kv_dtype == "bf16" else "e4m3 cache, f16 products",
            "data": "synthetic",
            "config": arm_config(wl, args, world, share),
            "legs": legs, "roofline": roof,
            "gpu_launches": path.launches_per_step() * args.steps,
            "clocks": clocks}

    if rank == 0 and world == 1 and args.config == 5 and not args.no_sub_configs:
        # the pages' own two shapes (q = k = 1024 prefill; batched decode) and the chunked
        # varlen prefill, each timed on its own (L2 flushed before every call)
        line["configs"] = run_sub_configs(args, device, peaks, peak_kind,
                                          with_oracle=not args.no_cpu_baseline)
    if rank == 0 and not args.no_e2e:
        line["e2e"] = run_e2e(path, args, world)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"], line["parity_sample"] = run_cpu_baseline(path, args)
        if args.kv_dtype == "fp8":  # the oracle sample reads the bf16 pools
            line["parity_sample"]["note"] = "vs the bf16 cache: includes E4M3 quantisation"
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


SUB_CONFIGS = (2, 3, 4)


def time_cold_calls(path, leg, steps, warmup, flush):
    """Device time of single calls with L2 flushed before each: events on the launching
    stream bracket every call; the flush runs before the first event of each pair."""
    stream = torch.cuda.current_stream(path.device)
    for _ in range(warmup):
        path.run_leg(leg)
    torch.cuda.synchronize()
    pairs = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        path.run_leg(leg)
        e1.record(stream)
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    cold = [a.elapsed_time(b) for a, b in pairs]
    # back to back, no flush: what a caller issuing calls in a loop sees (host launch
    # cost included when it exceeds the device time)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        path.run_leg(leg)
    e1.record(stream)
    torch.cuda.synchronize()
    b2b = e0.elapsed_time(e1) / steps
    # cold inside a stream of work: `steps` x (flush, call) between one event pair, less
    # `steps` flushes alone.  An event pair around a lone call also holds the launch of
    # the call, which the GPU front end only starts once the first event is written;
    # in a stream of kernels that launch overlaps the work before it.
    def loop(with_call):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            flush.zero_()
            if with_call:
                path.run_leg(leg)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps
    in_stream = statistics.median(loop(True) - loop(False) for _ in range(3))
    return (statistics.mean(cold), statistics.median(cold), min(cold), b2b, in_stream)


def run_sub_configs(args, device, peaks, peak_kind, with_oracle=True):
    """One record per config of SUB_CONFIGS: ms per call, rate and its fraction of the
    measured peak, and (cpu_baseline leg) the oracle's time on a bounded sample of the
    same call plus a parity check of the GPU outputs on the sampled rows."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    steps, warmup = max(args.steps, 10), max(args.warmup, 3)
    recs = {}
    for c in SUB_CONFIGS:
        wl = synth.make_workload(c, device=str(device))
        path = Path(wl, device, args.kv_dtype, share=False)
        leg = path.legs[0]
        b = leg["batch"]
        mean_ms, med_ms, min_ms, b2b_ms, stream_ms = time_cold_calls(path, leg, steps, warmup,
                                                                     flush)
        assert sa.seg_attn_take_device_error() == 0
        rec = {"workload": workload_name(wl), "mode": b.mode, "ms": mean_ms,
               "ms_median": med_ms, "ms_min": min_ms, "ms_back_to_back": b2b_ms,
               "ms_cold_in_stream": stream_ms,
               "launches": leg["launches"], "steps": steps,
               "l2": "flushed before every timed call (256 MB write)"}
        if leg["mode"] == sa.MODE_PREFILL:
            f = prefill_flops(b, wl)
            tf = f / (mean_ms * 1e-3) / 1e12
            rec.update({"flops": f, "tflops": tf, "frac_burst": tf / peaks["bf16_tflops"],
                        "frac_sustained": tf / peaks["bf16_tflops_sustained"],
                        "tflops_back_to_back": f / (b2b_ms * 1e-3) / 1e12,
                        "tflops_cold_in_stream": f / (stream_ms * 1e-3) / 1e12,
                        "frac_burst_cold_in_stream":
                            f / (stream_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                        "peak_kind": f"{peak_kind} burst bf16"})
        else:
            kvb = 1 if args.kv_dtype == "fp8" else 2
            by = decode_bytes(b, wl, leg["tab"].desc.table_bytes, kvb)
            gbs = by / (mean_ms * 1e-3) / 1e9
            rec.update({"bytes": by, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                        "gbs_cold_in_stream": by / (stream_ms * 1e-3) / 1e9,
                        "tflops": decode_flops(b, wl) / (mean_ms * 1e-3) / 1e12,
                        "peak_kind": f"{peak_kind} copy bandwidth"})
        if with_oracle:
            rows = {2: 1024, 3: 1024, 4: 512}[c]
            fl, sec, desc, results = oracle_sample(wl, wl.batches, [rows], rng_seed=4321 + c)
            worst = {"max_abs": 0.0, "mean_abs": 0.0, "lse_rel": 0.0, "rows": rows}
            for bi, toks, heads, o, l in results:
                go = leg["out"][toks.to(device), heads.to(device)].double().cpu()
                gl = leg["lse"][toks.to(device), heads.to(device)].double().cpu()
                err = (go - o).abs()
                worst["max_abs"] = max(worst["max_abs"], float(err.max()))
                worst["mean_abs"] = max(worst["mean_abs"], float(err.mean()))
                worst["lse_rel"] = max(worst["lse_rel"],
                                       float(((gl - l).abs() / l.abs().clamp(min=1)).max()))
            rec["parity_sample"] = worst
            rec["cpu_baseline"] = {"value": fl / sec / 1e12, "unit": "TFLOP/s",
                                   "cores": cpu_cores(), "kind": "oracle", "sample": desc,
                                   "seconds": sec}
        recs[str(c)] = rec
        del path, leg, wl, b
        torch.cuda.empty_cache()
    return recs


def time_plain_legs(wl, device, args):
    """Per-leg ms of the same workload with plain (unshared) tables, for comparison."""
    plain = Path(wl, device, args.kv_dtype, share=False)
    stream = torch.cuda.current_stream(device)
    for _ in range(args.warmup):
        for leg in plain.legs:
            plain.run_leg(leg)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(plain.legs) + 1)]
    tot = [0.0] * len(plain.legs)
    for _ in range(args.steps):
        ev[0].record(stream)
        for i, leg in enumerate(plain.legs):
            plain.run_leg(leg)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        for i in range(len(plain.legs)):
            tot[i] += ev[i].elapsed_time(ev[i + 1])
    return [t / args.steps for t in tot]


def run_e2e(path, args, world):
    """Same step through the public C-ABI calls with host buffers: every step copies its inputs
    (queries, both pools, tables) from pinned host memory and reads the outputs back."""
    wl = path.wl
    dev = path.device
    h_k = torch.empty(wl.k_pool.shape, dtype=wl.k_pool.dtype, pin_memory=True)
    h_v = torch.empty(wl.v_pool.shape, dtype=wl.v_pool.dtype, pin_memory=True)
    h_k.copy_(wl.k_pool)
    h_v.copy_(wl.v_pool)
    h_q = [torch.empty(l["batch"].q.shape, dtype=torch.bfloat16, pin_memory=True).copy_(l["batch"].q)
           for l in path.legs]
    h_out = [torch.empty(l["out"].shape, dtype=torch.bfloat16, pin_memory=True) for l in path.legs]
    h_lse = [torch.empty(l["lse"].shape, dtype=torch.float32, pin_memory=True) for l in path.legs]
    stream = torch.cuda.current_stream(dev)
    h2d = h_k.numel() * 2 + h_v.numel() * 2 + sum(q.numel() * 2 for q in h_q) + \
        sum(l["tab"].desc.table_bytes for l in path.legs)
    d2h = sum(o.numel() * 2 for o in h_out) + sum(l.numel() * 4 for l in h_lse)

    def step():
        wl.k_pool.copy_(h_k, non_blocking=True)
        wl.v_pool.copy_(h_v, non_blocking=True)
        for leg, hq in zip(path.legs, h_q):
            leg["batch"].q.copy_(hq, non_blocking=True)
            leg["tab"].device.copy_(leg["tab"].host, non_blocking=True)
        for leg in path.legs:
            path.run_leg(leg)
        for leg, ho, hl in zip(path.legs, h_out, h_lse):
            ho.copy_(leg["out"], non_blocking=True)
            hl.copy_(leg["lse"], non_blocking=True)

    n = max(1, min(args.steps, args.e2e_steps))
    step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(n):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / n
    flops = sum(prefill_flops(l["batch"], wl) if l["mode"] == sa.MODE_PREFILL else
                decode_flops(l["batch"], wl) for l in path.legs)
    return {"value": world * flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms,
            "steps": n}


def run_cpu_baseline(path, args):
    """The oracle on a bounded sample of the same workload (rank 0, N = 1), plus a parity
    spot check of the bench's own GPU outputs on the sampled rows."""
    wl = path.wl
    rows = [args.cpu_rows] * len(wl.batches)
    fl, sec, desc, results = oracle_sample(wl, wl.batches, rows, rng_seed=1234)
    worst = {"max_abs": 0.0, "mean_abs": 0.0, "lse_rel": 0.0}
    for bi, toks, heads, o, l in results:
        leg = path.legs[bi]
        go = leg["out"][toks.to(path.device), heads.to(path.device)].double().cpu()
        gl = leg["lse"][toks.to(path.device), heads.to(path.device)].double().cpu()
        err = (go - o).abs()
        worst["max_abs"] = max(worst["max_abs"], float(err.max()))
        worst["mean_abs"] = max(worst["mean_abs"], float(err.mean()))
        worst["lse_rel"] = max(worst["lse_rel"],
                               float(((gl - l).abs() / l.abs().clamp(min=1)).max()))
    base = {"value": fl / sec / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": desc, "seconds": sec}
    return base, worst


def run_kv_append(args):
    """Bandwidth of seg_attn_kv_append: 262144 new tokens (64/8 heads, d 128) scattered to
    slots handed out by the segment allocator for 256 sequences; prints its own JSON line."""
    device = torch.device("cuda", 0)
    hkv, d, n_seq, per_seq = 8, 128, 256, 1024
    S = int(1.1 * n_seq * per_seq)
    pool = sa.SegPool(S)
    g = torch.Generator(device=device).manual_seed(0)
    slots = torch.cat([torch.from_numpy(pool.append(s, per_seq)) for s in range(n_seq)]).to(device)
    n = slots.numel()
    k_pool = torch.empty(S, hkv, d, dtype=torch.bfloat16, device=device)
    v_pool = torch.empty_like(k_pool)
    k_new = torch.randn(n, hkv, d, generator=g, device=device).to(torch.bfloat16)
    v_new = torch.randn(n, hkv, d, generator=g, device=device).to(torch.bfloat16)
    for _ in range(args.warmup):
        sa.seg_attn_kv_append(k_new, v_new, slots, k_pool, v_pool)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        sa.seg_attn_kv_append(k_new, v_new, slots, k_pool, v_pool)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / args.steps
    by = 2 * 2 * n * hkv * d * 2 + 4 * n  # K and V read + written, plus the slot array
    peaks, kind = load_peaks()
    ok = torch.equal(k_pool[slots.long()].view(torch.int16), k_new.view(torch.int16))
    print(json.dumps({"metric": "kv append HBM GB/s", "value": by / (ms * 1e-3) / 1e9,
                      "unit": "GB/s", "ms_per_step": ms, "steps": args.steps,
                      "frac_hbm": by / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "bytes": by,
                      "tokens": n, "bit_exact": bool(ok),
                      "device_error": sa.seg_attn_take_device_error()}), flush=True)
    return 0


def la_algorithmic(w):
    """(bytes, flops) a linear-attention call must move / do: q, k, v, g read, out written,
    states read and written once; prefill flops of the chunked form (Q K^T, P V, Q S and
    the chunk state K'^T V per 128-token chunk)."""
    T, H, d = w.q.shape
    B = len(w.q_lens)
    state = d * d * 4
    by = 4 * T * H * d * 2 + T * H * 4
    by += sum(state * H for s in w.in_slot if s >= 0) + sum(state * H for s in w.out_slot if s >= 0)
    if w.mode == "decode":
        return by, 6.0 * B * H * d * d
    fl = 0.0
    for n in w.q_lens:
        for t0 in range(0, n, 128):
            c = min(128, n - t0)
            fl += H * (4.0 * c * c * d + 4.0 * c * d * d)
    return by, fl


def run_linear(args):
    """Segment linear attention on the shapes of the Flood README "Seg-linear-attn" table;
    one JSON line with the per-call latency of each shape."""
    import oracle
    device = torch.device("cuda", 0)
    peaks, kind = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    res = {}
    for name in synth.LA_CONFIGS:
        w = synth.make_la_workload(name, device=str(device))
        mode = sa.MODE_PREFILL if w.mode == "prefill" else sa.MODE_DECODE
        tab = sa.LATable.build(w.q_lens if mode == sa.MODE_PREFILL else None, w.in_slot,
                               w.out_slot, w.state_pool.shape[0], mode, w.heads, w.head_dim,
                               pin=True).to(device)
        out = torch.empty_like(w.q)
        pool0 = w.state_pool.clone()
        ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device=device)
              if tab.workspace_bytes else None)

        def call():
            if mode == sa.MODE_PREFILL:
                sa.seg_la_prefill(w.q, w.k, w.v, w.g, out, w.state_pool, tab.device, tab.desc,
                                  w.scale, ws)
            else:
                sa.seg_la_decode(w.q, w.k, w.v, w.g, out, w.state_pool, tab.device, tab.desc,
                                 w.scale)
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        times = []
        for _ in range(args.steps):
            flush.zero_()  # L2 cold for every call
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3)
        assert sa.seg_attn_take_device_error() == 0
        us = statistics.median(times)
        by, fl = la_algorithmic(w)
        gbs = by / (us * 1e-6) / 1e9
        entry = {"us": us, "us_min": min(times), "launches": 3 if mode == sa.MODE_PREFILL else 1,
                 "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                              "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "bytes": by,
                              "traffic": None},
                 "tflops": fl / (us * 1e-6) / 1e12}
        # parity spot check of this run's outputs (first request / first rows), state reset
        w.state_pool.copy_(pool0)
        call()
        torch.cuda.synchronize()
        n = min(w.q_lens[0], 256) if mode == sa.MODE_PREFILL else 1
        s0 = w.in_slot[0]
        st = pool0[s0:s0 + 1].cpu() if s0 >= 0 else None
        args_o = ([n], w.q[:n].cpu(), w.k[:n].cpu(), w.v[:n].cpu(), w.g[:n].cpu(), w.scale, st,
                  [0 if s0 >= 0 else -1])
        t0 = time.perf_counter()
        ro, _ = oracle.linear_attention(*args_o)
        secs = time.perf_counter() - t0
        err = (out[:n].double().cpu() - ro).abs()
        entry["parity_sample"] = {"rows": n, "max_abs_over_rms": float(err.max() / ro.pow(2).mean().sqrt())}
        entry["cpu_baseline"] = {"value": secs * 1e6 * sum(w.q_lens) / n,
                                 "unit": "us (oracle, scaled from the sample)",
                                 "cores": cpu_cores(), "kind": "oracle",
                                 "sample": f"request 0, first {n} tokens, all heads"}
        res[name] = entry
        del w, tab, out, pool0, ws
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "seg-linear-attn latency per call (16/16 heads, d 128)",
                      "unit": "us", "higher_is_better": False, "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "dtype": "bf16 (fp32 state)", "data": "synthetic",
                      "config": {"workload": "Seg-linear-attn table shapes",
                                 "l2": "flushed before every timed call (256 MB write)"},
                      "peak_kind": f"{kind} copy bandwidth", "shapes": res}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=5, choices=[1, 2, 3, 4, 5, 6, 7])
    ap.add_argument("--share-prefix", dest="share_prefix", action="store_true", default=None,
                    help="build tables with SEG_ATTN_SHARE_PREFIX (default: configs 6 and 7)")
    ap.add_argument("--no-share-prefix", dest="share_prefix", action="store_false")
    ap.add_argument("--ref-rows", type=int, default=48,
                    help="oracle rows per batch per step (bounded CPU sample)")
    ap.add_argument("--cpu-rows", type=int, default=1536,
                    help="oracle rows per batch for the cpu_baseline leg of our arm")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="KV cache type of every leg (fp8: E4M3 with per-kv-head scales)")
    ap.add_argument("--kv-append", action="store_true",
                    help="measure the KV-append kernel instead of the attention step")
    ap.add_argument("--linear", action="store_true",
                    help="measure segment linear attention on the Seg-linear-attn table shapes")
    ap.add_argument("--context-scale", type=float, default=1.0,
                    help="shorten the long-context mix (profiling captures only; 1.0 = as specified)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-configs", action="store_true",
                    help="skip the per-config records of configs 2, 3 and 4 (default run only)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.kv_append:
        return run_kv_append(args)
    if args.linear:
        return run_linear(args)
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
