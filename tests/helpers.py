"""Shared test helpers: run the CUDA path through the C ABI, compare with the oracle."""
from __future__ import annotations

import math
import random

import numpy as np
import torch

import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import synth

# Tolerances (bf16 inputs, fp32 accumulation, bf16 output) against the fp64 oracle.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_REL = 1e-3


def run_cuda(q, k_pool, v_pool, q_lens, seg_starts, seg_lens, num_slots, causal, mode, scale,
             stream=None):
    """One call through the C ABI on device tensors; returns (out, lse, table)."""
    hq, d = q.shape[1], q.shape[2]
    hkv = k_pool.shape[1]
    tab = sa.SegTable.build(q_lens, seg_starts, seg_lens, num_slots, causal, mode, hq, hkv, d)
    tab.to(q.device)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((q.shape[0], hq), float("nan"), dtype=torch.float32, device=q.device)
    ws = None
    if tab.workspace_bytes:
        ws = torch.empty(tab.workspace_bytes, dtype=torch.uint8, device=q.device)
    fn = sa.seg_attn_prefill if (mode & 0xff) == sa.MODE_PREFILL else sa.seg_attn_decode
    fn(q, k_pool, v_pool, out, lse, tab.device, tab.desc, scale, ws, stream)
    return out, lse, tab


def run_batch(wl, batch, stream=None):
    mode = sa.MODE_PREFILL if batch.mode == "prefill" else sa.MODE_DECODE
    return run_cuda(batch.q, wl.k_pool, wl.v_pool, batch.q_lens if mode == sa.MODE_PREFILL else None,
                    batch.seg_starts, batch.seg_lens, wl.num_slots, batch.causal, mode, wl.scale,
                    stream)


def compare(out, lse, ref_out, ref_lse, what=""):
    """Element-wise comparison against the oracle; returns the error summary."""
    o = out.detach().double().cpu()
    l = lse.detach().double().cpu()
    assert o.shape == ref_out.shape, (o.shape, ref_out.shape)
    assert torch.isfinite(o).all(), f"{what}: non-finite output"
    err = (o - ref_out).abs()
    max_abs, mean_abs = float(err.max()) if err.numel() else 0.0, float(err.mean()) if err.numel() else 0.0
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(l), fin), f"{what}: lse finiteness differs"
    assert torch.equal(l[~fin], ref_lse[~fin]), f"{what}: -inf lse rows differ"
    lerr = ((l[fin] - ref_lse[fin]).abs() / ref_lse[fin].abs().clamp(min=1.0))
    lse_rel = float(lerr.max()) if lerr.numel() else 0.0
    summary = dict(max_abs=max_abs, mean_abs=mean_abs, lse_rel=lse_rel)
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs}"
    assert mean_abs <= MEAN_ABS, f"{what}: mean-abs {mean_abs}"
    assert lse_rel <= LSE_REL, f"{what}: lse rel {lse_rel}"
    return summary


def compact_requests(wl, batch, req_ids):
    """CPU copy of a subset of requests with a pool holding only their segments.

    Moving segments to other slots leaves the result unchanged (an invariance
    the oracle tests pin), so the oracle can run on the compact pool.
    """
    seg_starts, seg_lens, slots = [], [], []
    pos = 0
    for r in req_ids:
        ss, ll = [], []
        for s, l in zip(batch.seg_starts[r], batch.seg_lens[r]):
            ss.append(pos)
            ll.append(l)
            slots.append(torch.arange(s, s + l))
            pos += l
        seg_starts.append(ss)
        seg_lens.append(ll)
    idx = torch.cat(slots) if slots else torch.zeros(0, dtype=torch.long)
    dev = wl.k_pool.device
    k = wl.k_pool[idx.to(dev)].cpu()
    v = wl.v_pool[idx.to(dev)].cpu()
    q_off = np.concatenate([[0], np.cumsum(batch.q_lens)])
    q_rows = torch.cat([torch.arange(q_off[r], q_off[r + 1]) for r in req_ids])
    q = batch.q[q_rows.to(batch.q.device)].cpu()
    q_lens = [batch.q_lens[r] for r in req_ids]
    return dict(q=q, k_pool=k, v_pool=v, q_lens=q_lens, seg_starts=seg_starts, seg_lens=seg_lens,
                q_rows=q_rows)


def random_case(seed, batch, hq, hkv, d, causal, max_k, nseg_max=4, q_mode="chunk",
                device="cuda", extra_slots=97):
    """Seeded small case with NaN-filled free slots (values drawn on the CPU)."""
    g = torch.Generator().manual_seed(seed)
    k_lens = torch.randint(1, max_k + 1, (batch,), generator=g).tolist()
    if q_mode == "full":
        q_lens = list(k_lens)
    elif q_mode == "decode":
        q_lens = [1] * batch
    else:
        q_lens = [int(torch.randint(0, k + 1, (1,), generator=g)) for k in k_lens]
    seg_lens = [synth.split_uniform_cuts(k, int(torch.randint(1, nseg_max + 1, (1,), generator=g)), g)
                for k in k_lens]
    flat = [x for s in seg_lens for x in s]
    slots = sum(flat) + extra_slots
    starts = synth.place_segments(flat, slots, g)
    it = iter(starts)
    seg_starts = [[next(it) for _ in s] for s in seg_lens]
    q = torch.randn(sum(q_lens), hq, d, generator=g).to(torch.bfloat16)
    k = torch.full((slots, hkv, d), float("nan")).to(torch.bfloat16)
    v = torch.full((slots, hkv, d), float("nan")).to(torch.bfloat16)
    for ss, ll in zip(seg_starts, seg_lens):
        for s, l in zip(ss, ll):
            k[s:s + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
            v[s:s + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
    return dict(q_lens=q_lens, seg_starts=seg_starts, seg_lens=seg_lens, q=q, k_pool=k, v_pool=v,
                num_slots=slots, scale=1.0 / math.sqrt(d), causal=causal)


def slots_of(starts, lens):
    return [s + t for s, l in zip(starts, lens) for t in range(l)]


def shared_case(seed, B, decode, max_prefix=1200):
    """Requests drawn from a few prefix trees: each shares a random-length prefix with
    its predecessor (sometimes re-cut into other segments), then has its own keys."""
    rnd = random.Random(seed)
    pool_next = [0]

    def fresh(n):
        s = pool_next[0] + rnd.randint(0, 5)
        pool_next[0] = s + n
        return (s, n)

    reqs = []
    prev = None
    for r in range(B):
        segs = []
        if prev is not None and rnd.random() < 0.75:
            # take a prefix of the previous request's slots, maybe cut differently
            ps = slots_of(*prev)
            take = rnd.randint(0, len(ps))
            run_start, run_len = None, 0
            for x in ps[:take]:
                if run_start is not None and x == run_start + run_len and rnd.random() < 0.97:
                    run_len += 1
                else:
                    if run_start is not None:
                        segs.append((run_start, run_len))
                    run_start, run_len = x, 1
            if run_start is not None:
                segs.append((run_start, run_len))
        else:
            segs.append(fresh(rnd.randint(0, max_prefix)))
        for _ in range(rnd.randint(0 if segs else 1, 3)):
            segs.append(fresh(rnd.randint(1, 300)))
        segs = [s for s in segs if s[1] > 0] or [fresh(1)]
        starts, lens = [s for s, _ in segs], [l for _, l in segs]
        reqs.append((starts, lens))
        prev = (starts, lens)
    k = [sum(l) for _, l in reqs]
    if decode:
        q = [1] * B
    else:
        q = [rnd.randint(0, min(kk, 40)) for kk in k]
    return reqs, q, pool_next[0] + 10


def shared_values(reqs, q_lens, num_slots, hq, hkv, d, seed, device="cuda"):
    """Q and pools for a shared_case: the slots any request uses get N(0,1) bf16 values,
    every other slot NaN (drawn on the CPU)."""
    g = torch.Generator().manual_seed(seed)
    live = torch.zeros(num_slots, dtype=torch.bool)
    for starts, lens in reqs:
        for s, l in zip(starts, lens):
            live[s:s + l] = True
    k = torch.full((num_slots, hkv, d), float("nan"))
    v = torch.full((num_slots, hkv, d), float("nan"))
    n = int(live.sum())
    k[live] = torch.randn(n, hkv, d, generator=g)
    v[live] = torch.randn(n, hkv, d, generator=g)
    q = torch.randn(sum(q_lens), hq, d, generator=g)
    return dict(q=q.to(torch.bfloat16), k_pool=k.to(torch.bfloat16), v_pool=v.to(torch.bfloat16),
                q_lens=list(q_lens), seg_starts=[s for s, _ in reqs],
                seg_lens=[l for _, l in reqs], num_slots=num_slots, scale=1.0 / math.sqrt(d))
