"""Shared test helpers: run the CUDA path through the C ABI, compare with the oracle."""
from __future__ import annotations

import math

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
    fn = sa.seg_attn_prefill if mode == sa.MODE_PREFILL else sa.seg_attn_decode
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
