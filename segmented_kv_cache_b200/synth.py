"""Seeded synthetic workloads for SegmentAttention.

This module only draws inputs: request lengths, segment lists, slot placement
and the Q / K / V values.  It holds no attention arithmetic, so both the CUDA
path and the fp64 oracle can take their inputs from it.

The workloads follow the kernel benchmark of the Flood README ("Kernels >
Seg-attn": 64 query heads, 8 kv heads, head_dim 128) and its segmentable
KV cache ("Introduction": each request's cache is a few contiguous runs of
token slots in a shared pool instead of fixed pages).

Draw order, fixed for every config: lengths -> segment counts -> cut points
-> placement -> Q -> K -> V.  Lengths, counts, cut points and placement always
come from a CPU ``torch.Generator`` seeded with the config seed, so the table
structure does not depend on the device.  Values come from a generator on the
requested device seeded with the same seed; large pools are drawn on the GPU
because drawing billions of normals on the host takes minutes.  Free pool
slots are filled with NaN so that a read outside the segment lists poisons
the output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

__all__ = ["Batch", "Workload", "make_workload", "CONFIG_NAMES", "split_uniform_cuts",
           "place_segments", "fp8_pools", "LAWorkload", "make_la_workload", "LA_CONFIGS"]

CONFIG_NAMES = {
    1: "tiny causal prefill (2 req, q=k=16/33, 4/1 heads, d64)",
    2: "pages-shaped prefill (1 req, q=k=1024, 64/8 heads, d128)",
    3: "chunked prefill varlen (16 req, 2048 new tokens, prior 0-8192)",
    4: "batched decode (128 req, k 1024-32768)",
    5: "long-context mix (8 decode at k=131072 + 1 prefill chunk 2048 over 131072)",
    6: "shared-prefix decode (8 groups x 8 req, prefix 8192-32768 + own 512-4096)",
    7: "shared-prefix chunked prefill (4 groups x 8 req, prefix 4096-16384, chunks 4-32)",
}


@dataclass
class Batch:
    """One call's worth of requests over the shared pool."""
    mode: str                      # "prefill" or "decode"
    q_lens: List[int]
    seg_starts: List[List[int]]    # per request, logical (list) order
    seg_lens: List[List[int]]
    causal: bool
    q: Optional[torch.Tensor] = None   # bf16 [sum(q_lens), Hq, d]

    @property
    def batch(self) -> int:
        return len(self.q_lens)

    @property
    def k_lens(self) -> List[int]:
        return [sum(s) for s in self.seg_lens]

    @property
    def total_q(self) -> int:
        return sum(self.q_lens)

    def flat_segments(self):
        counts = [len(s) for s in self.seg_starts]
        starts = [x for s in self.seg_starts for x in s]
        lens = [x for s in self.seg_lens for x in s]
        return counts, starts, lens


@dataclass
class Workload:
    config: int
    name: str
    q_heads: int
    kv_heads: int
    head_dim: int
    num_slots: int
    scale: float
    batches: List[Batch]
    k_pool: Optional[torch.Tensor] = None   # bf16 [S, Hkv, d]
    v_pool: Optional[torch.Tensor] = None
    live: Optional[torch.Tensor] = field(default=None, repr=False)  # bool [S]


def split_uniform_cuts(total: int, nseg: int, gen: torch.Generator) -> List[int]:
    """Split ``total`` tokens into ``nseg`` positive lengths at distinct uniform cut points."""
    if total <= 0:
        return []
    nseg = max(1, min(nseg, total))
    if nseg == 1:
        return [total]
    cuts = (torch.randperm(total - 1, generator=gen)[: nseg - 1] + 1).sort().values.tolist()
    edges = [0] + cuts + [total]
    return [edges[i + 1] - edges[i] for i in range(nseg)]


def place_segments(all_lens: List[int], num_slots: int, gen: torch.Generator) -> List[int]:
    """Random non-overlapping placement: shuffle every segment of every request,
    cut the free slots into nseg+1 gaps at sorted uniform points, then lay gaps
    and segments out alternately.  Returns the start slot of each segment."""
    nseg = len(all_lens)
    live = sum(all_lens)
    free = num_slots - live
    assert free >= 0, "pool too small"
    order = torch.randperm(nseg, generator=gen).tolist()
    cuts = torch.randint(0, free + 1, (nseg,), generator=gen).sort().values.tolist()
    gaps = [cuts[0]] + [cuts[i] - cuts[i - 1] for i in range(1, nseg)]
    starts = [0] * nseg
    pos = 0
    for i, s in enumerate(order):
        pos += gaps[i]
        starts[s] = pos
        pos += all_lens[s]
    assert pos <= num_slots
    return starts


def _values(shape, gen, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def _pool_values(num_slots, kv_heads, head_dim, live, gen, device, std):
    """Pool values drawn in slices (bounded temporary memory), free slots NaN."""
    pool = torch.empty((num_slots, kv_heads, head_dim), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 26) // (kv_heads * head_dim))
    for a in range(0, num_slots, step):
        b = min(num_slots, a + step)
        pool[a:b] = _values((b - a, kv_heads, head_dim), gen, device, std)
    pool[~live.to(device)] = float("nan")
    return pool


def _structure(cfg: int, gen: torch.Generator, context_scale: float = 1.0):
    """Lengths, segment counts and cut points of each config (no values).

    ``context_scale`` shortens the long-context mix (config 5) for profiling
    runs that must stay small; every other config ignores it."""
    if cfg == 1:
        q_lens = [16, 33]
        seg_lens = [[8, 8], [17, 16]]
        return dict(q_heads=4, kv_heads=1, head_dim=64, num_slots=128,
                    batches=[("prefill", q_lens, seg_lens, True)], qk_std=1.0)
    if cfg == 2:
        return dict(q_heads=64, kv_heads=8, head_dim=128, num_slots=65536,
                    batches=[("prefill", [1024], [[256, 256, 256, 256]], True)], qk_std=1.0)
    if cfg == 3:
        B = 16
        prior = torch.randint(0, 8193, (B,), generator=gen).tolist()
        q_lens = torch.bincount(torch.randint(0, B, (2048,), generator=gen), minlength=B).tolist()
        k_lens = [p + q for p, q in zip(prior, q_lens)]
        nsegs = torch.randint(1, 7, (B,), generator=gen).tolist()
        seg_lens = [split_uniform_cuts(k, n, gen) for k, n in zip(k_lens, nsegs)]
        return dict(q_heads=64, kv_heads=8, head_dim=128, num_slots=262144,
                    batches=[("prefill", q_lens, seg_lens, True)], qk_std=1.0)
    if cfg == 4:
        B = 128
        k_lens = torch.randint(1024, 32769, (B,), generator=gen).tolist()
        nsegs = torch.randint(1, 9, (B,), generator=gen).tolist()
        seg_lens = [split_uniform_cuts(k, n, gen) for k, n in zip(k_lens, nsegs)]
        slots = math.ceil(1.1 * sum(k_lens))
        return dict(q_heads=64, kv_heads=8, head_dim=128, num_slots=slots,
                    batches=[("decode", [1] * B, seg_lens, True)], qk_std=1.0)
    if cfg == 5:
        ctx = max(1024, int(131072 * context_scale))
        k_dec = [ctx] * 8
        k_pre = [ctx + 2048]
        nsegs = torch.randint(4, 17, (9,), generator=gen).tolist()
        lens_all = [split_uniform_cuts(k, n, gen) for k, n in zip(k_dec + k_pre, nsegs)]
        slots = math.ceil(1.1 * (sum(k_dec) + sum(k_pre)))
        return dict(q_heads=64, kv_heads=8, head_dim=128, num_slots=slots,
                    batches=[("decode", [1] * 8, lens_all[:8], True),
                             ("prefill", [2048], lens_all[8:], True)], qk_std=0.5)
    if cfg in (6, 7):
        return _shared_structure(cfg, gen)
    raise ValueError(f"unknown config {cfg}")


def _shared_structure(cfg: int, gen: torch.Generator):
    """Requests in groups of consecutive requests that share a prefix (prefix caching):
    every member's segment list starts with the group's prefix segments (the same
    slots), then lists its own segments.
      6: decode, 8 groups x 8 requests; prefix U{8192..32768} keys in U{1..4}
         segments; each request's own keys U{512..4096} in U{1..4} segments.
      7: causal chunked prefill, 4 groups x 8 requests; prefix U{4096..16384} in
         U{1..4} segments; each request's own prior context U{0..1024} plus a new
         chunk of U{4..32} queries (short chunks: multi-token verification, short
         turns), in U{1..3} segments.
    Draw order: per group the prefix length, its segment count and cuts, then per
    member its own lengths, segment count and cuts."""
    groups, members = (8, 8) if cfg == 6 else (4, 8)
    unique, q_lens, seg_ids = [], [], []
    for _ in range(groups):
        if cfg == 6:
            P = int(torch.randint(8192, 32769, (1,), generator=gen))
        else:
            P = int(torch.randint(4096, 16385, (1,), generator=gen))
        n = int(torch.randint(1, 5, (1,), generator=gen))
        prefix_ids = []
        for ln in split_uniform_cuts(P, n, gen):
            prefix_ids.append(len(unique))
            unique.append(ln)
        for _ in range(members):
            if cfg == 6:
                q, own = 1, int(torch.randint(512, 4097, (1,), generator=gen))
                n_own = int(torch.randint(1, 5, (1,), generator=gen))
            else:
                prior = int(torch.randint(0, 1025, (1,), generator=gen))
                q = int(torch.randint(4, 33, (1,), generator=gen))
                own = prior + q
                n_own = int(torch.randint(1, 4, (1,), generator=gen))
            ids = list(prefix_ids)
            for ln in split_uniform_cuts(own, n_own, gen):
                ids.append(len(unique))
                unique.append(ln)
            q_lens.append(q)
            seg_ids.append(ids)
    slots = math.ceil(1.1 * sum(unique))
    mode = "decode" if cfg == 6 else "prefill"
    return dict(q_heads=64, kv_heads=8, head_dim=128, num_slots=slots, unique=unique,
                batches=[(mode, q_lens, seg_ids, True)], qk_std=1.0)


def make_workload(cfg: int, device: str = "cpu", values: bool = True,
                  seed: Optional[int] = None, context_scale: float = 1.0) -> Workload:
    """Build config ``cfg`` (1..7).  Seed defaults to cfg - 1."""
    seed = cfg - 1 if seed is None else seed
    gen = torch.Generator(device="cpu").manual_seed(seed)
    st = _structure(cfg, gen, context_scale)
    batches = []
    if "unique" in st:
        # segments listed by id into one list of distinct segments (shared prefixes)
        unique = st["unique"]
        for mode, q_lens, seg_ids, causal in st["batches"]:
            batches.append(Batch(mode=mode, q_lens=list(q_lens), seg_starts=[],
                                 seg_lens=[[unique[i] for i in ids] for ids in seg_ids],
                                 causal=causal))
        starts = place_segments(unique, st["num_slots"], gen)
        for b, (_, _, seg_ids, _) in zip(batches, st["batches"]):
            b.seg_starts = [[starts[i] for i in ids] for ids in seg_ids]
    else:
        all_lens = []
        for mode, q_lens, seg_lens, causal in st["batches"]:
            batches.append(Batch(mode=mode, q_lens=list(q_lens), seg_starts=[],
                                 seg_lens=seg_lens, causal=causal))
            for s in seg_lens:
                all_lens.extend(s)
        starts = place_segments(all_lens, st["num_slots"], gen)
        it = iter(starts)
        for b in batches:
            b.seg_starts = [[next(it) for _ in s] for s in b.seg_lens]
    live = torch.zeros(st["num_slots"], dtype=torch.bool)
    for b in batches:
        for ss, ll in zip(b.seg_starts, b.seg_lens):
            for s, l in zip(ss, ll):
                live[s:s + l] = True
    wl = Workload(config=cfg, name=CONFIG_NAMES[cfg], q_heads=st["q_heads"],
                  kv_heads=st["kv_heads"], head_dim=st["head_dim"], num_slots=st["num_slots"],
                  scale=1.0 / math.sqrt(st["head_dim"]), batches=batches, live=live)
    if values:
        vgen = torch.Generator(device=device).manual_seed(seed)
        for b in batches:
            b.q = _values((b.total_q, wl.q_heads, wl.head_dim), vgen, device, st["qk_std"])
        wl.k_pool = _pool_values(wl.num_slots, wl.kv_heads, wl.head_dim, live, vgen, device,
                                 st["qk_std"])
        wl.v_pool = _pool_values(wl.num_slots, wl.kv_heads, wl.head_dim, live, vgen, device, 1.0)
    return wl


def fp8_pools(k_pool: torch.Tensor, v_pool: torch.Tensor):
    """E4M3 copies of bf16 pools for the FP8 KV-cache variant: per-kv-head scales so the
    largest live magnitude maps to 448, codes from torch's float8_e4m3fn cast (free NaN
    slots stay NaN codes).  Returns (k8, v8 as uint8 views, k_scale, v_scale fp32)."""
    def one(pool):
        amax = torch.nan_to_num(pool.float(), nan=0.0).abs().amax(dim=(0, 2)).clamp(min=1e-30)
        scale = (amax / 448.0).float()
        codes = (pool.float() / scale.view(1, -1, 1)).clamp(-448, 448).to(torch.float8_e4m3fn)
        return codes.view(torch.uint8), scale
    k8, ks = one(k_pool)
    v8, vs = one(v_pool)
    return k8, v8, ks, vs


# --------------------------------------------------------------------------- linear attention
# Shapes of the Flood README "Kernels > Seg-linear-attn" table: 16 heads, 16 kv
# heads, head_dim 128; prefill batch 1 and 2 at 1024 tokens, decode batch 64 and 256.
LA_CONFIGS = {
    "la-prefill-1x1024": dict(mode="prefill", batch=1, q_len=1024, seed=11),
    "la-prefill-2x1024": dict(mode="prefill", batch=2, q_len=1024, seed=12),
    "la-decode-64": dict(mode="decode", batch=64, q_len=1, seed=13),
    "la-decode-256": dict(mode="decode", batch=256, q_len=1, seed=14),
}


@dataclass
class LAWorkload:
    """One call of segment linear attention: packed tokens of every request, the state
    pool and each request's slots (in_slot -1: the request starts from a zero state)."""
    name: str
    mode: str
    heads: int
    head_dim: int
    q_lens: List[int]
    q: torch.Tensor          # bf16 [T, H, d]
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor          # fp32 [T, H], log of the per-token decay
    state_pool: torch.Tensor  # fp32 [num_state_slots, H, d, d]
    in_slot: List[int]
    out_slot: List[int]
    scale: float


def make_la_workload(name: str, device: str = "cpu", seed: Optional[int] = None,
                     heads: int = 16, head_dim: int = 128, q_lens: Optional[List[int]] = None,
                     fresh: Optional[bool] = None) -> LAWorkload:
    """Inputs of a linear-attention config (``LA_CONFIGS``) or, with ``q_lens`` given, of a
    custom batch.  q, k, v ~ N(0, 1) in bf16; g = log(sigmoid(x)) / 16 with x ~ N(0, 1)
    (per-token decay exp(g) in (0.94, 1)); the pool has 2 state slots per request, every
    state ~ 4 * N(0, 1) (the size a state reaches under that decay); decode requests read
    their state from a random slot and write it back there, prefill requests start from a
    zero state (``fresh``) and write a slot of their own.  Draw order: slots -> q -> k ->
    v -> g -> states, on a generator seeded with the config seed."""
    cfg = LA_CONFIGS.get(name, {})
    mode = cfg.get("mode", "prefill")
    if q_lens is None:
        q_lens = [cfg["q_len"]] * cfg["batch"]
    seed = cfg.get("seed", 0) if seed is None else seed
    fresh = (mode == "prefill") if fresh is None else fresh
    B = len(q_lens)
    gen = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(2 * B, generator=gen).tolist()
    out_slot = perm[:B]
    in_slot = [-1] * B if fresh else list(out_slot)
    vgen = torch.Generator(device=device).manual_seed(seed)
    T = sum(q_lens)
    q = _values((T, heads, head_dim), vgen, device)
    k = _values((T, heads, head_dim), vgen, device)
    v = _values((T, heads, head_dim), vgen, device)
    x = torch.randn((T, heads), generator=vgen, device=device, dtype=torch.float32)
    g = torch.nn.functional.logsigmoid(x) / 16.0
    states = torch.randn((2 * B, heads, head_dim, head_dim), generator=vgen, device=device,
                         dtype=torch.float32) * 4.0
    return LAWorkload(name=name, mode=mode, heads=heads, head_dim=head_dim, q_lens=list(q_lens),
                      q=q, k=k, v=v, g=g, state_pool=states, in_slot=in_slot, out_slot=out_slot,
                      scale=1.0 / math.sqrt(head_dim))
