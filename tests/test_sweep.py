"""Seeded sweep across every feature combination of the attention path, small cases
against the fp64 oracle: cache type (bf16 / E4M3) x prefill / decode x shared-prefix
planning on / off x head_dim x GQA group x causal.  The focused tests vary one feature
at a time; this crosses them."""
import math

import numpy as np
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import synth

from helpers import compare, shared_case, shared_values

pytestmark = pytest.mark.gpu

# the last shape of each: a GQA group above 8 (decode covers it with sibling CTAs)
HEADS = {64: [(8, 1), (16, 2), (32, 8), (32, 2)], 128: [(64, 8), (16, 4), (8, 8), (64, 1)]}


def _case(seed, decode, d, hq, hkv, shared):
    if shared:
        reqs, q_lens, S = shared_case(seed, B=6, decode=decode, max_prefix=1500)
        return shared_values(reqs, q_lens, S, hq, hkv, d, seed=seed + 5)
    rnd = np.random.default_rng(seed)
    B = int(rnd.integers(1, 6))
    k_lens = [int(rnd.integers(1, 1500)) for _ in range(B)]
    q_lens = [1 if decode else int(rnd.integers(0, k + 1)) for k in k_lens]
    g = torch.Generator().manual_seed(seed)
    seg_lens = [synth.split_uniform_cuts(k, int(rnd.integers(1, 5)), g) for k in k_lens]
    flat = [x for s in seg_lens for x in s]
    S = sum(flat) + 50
    starts = synth.place_segments(flat, S, g)
    it = iter(starts)
    seg_starts = [[next(it) for _ in s] for s in seg_lens]
    k = torch.full((S, hkv, d), float("nan"))
    v = torch.full((S, hkv, d), float("nan"))
    for ss, ll in zip(seg_starts, seg_lens):
        for s0, l in zip(ss, ll):
            k[s0:s0 + l] = torch.randn(l, hkv, d, generator=g)
            v[s0:s0 + l] = torch.randn(l, hkv, d, generator=g)
    q = torch.randn(sum(q_lens), hq, d, generator=g)
    return dict(q=q.to(torch.bfloat16), k_pool=k.to(torch.bfloat16), v_pool=v.to(torch.bfloat16),
                q_lens=q_lens, seg_starts=seg_starts, seg_lens=seg_lens, num_slots=S,
                scale=1.0 / math.sqrt(d))


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "e4m3"])
@pytest.mark.parametrize("decode", [False, True], ids=["prefill", "decode"])
@pytest.mark.parametrize("shared", [False, True], ids=["plain", "shared"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hi", [0, 1, 2, 3])
def test_sweep(fp8, decode, shared, d, hi):
    hq, hkv = HEADS[d][hi]
    seed = 1000 + 97 * hi + 13 * d + 7 * decode + 3 * shared + fp8
    case = _case(seed, decode, d, hq, hkv, shared)
    causal = decode or bool(seed % 3)
    mode = (sa.MODE_DECODE if decode else sa.MODE_PREFILL) | (sa.SHARE_PREFIX if shared else 0)
    tab = sa.SegTable.build(None if decode else case["q_lens"], case["seg_starts"],
                            case["seg_lens"], case["num_slots"], causal, mode, hq, hkv, d)
    tab.to("cuda")
    q = case["q"].cuda()
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device="cuda")
          if tab.workspace_bytes else None)
    if fp8:
        k8, v8, ks, vs = synth.fp8_pools(case["k_pool"], case["v_pool"])
        fn = sa.seg_attn_decode_fp8 if decode else sa.seg_attn_prefill_fp8
        fn(q, k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda(), out, lse, tab.device, tab.desc,
           case["scale"], ws)
        ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                            case["q"], k8, v8, ks, vs, case["scale"], causal)
    else:
        fn = sa.seg_attn_decode if decode else sa.seg_attn_prefill
        fn(q, case["k_pool"].cuda(), case["v_pool"].cuda(), out, lse, tab.device, tab.desc,
           case["scale"], ws)
        ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                        case["q"], case["k_pool"], case["v_pool"], case["scale"],
                                        causal)
    torch.cuda.synchronize()
    compare(out, lse, ref_o, ref_l,
            f"sweep {'e4m3' if fp8 else 'bf16'} {'decode' if decode else 'prefill'} "
            f"{'shared' if shared else 'plain'} d{d} {hq}/{hkv} causal={causal}")
    assert sa.seg_attn_take_device_error() == 0
