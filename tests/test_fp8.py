"""FP8 (E4M3) KV cache: quantising append (bit-exact) and decode parity against the
FP8 oracle path (same tolerances as the bf16 cache)."""
import math

import numpy as np
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import synth

from helpers import compact_requests, compare, random_case, shared_case, shared_values, slots_of

pytestmark = pytest.mark.gpu


def test_fp8_append_matches_torch_quantisation():
    g = torch.Generator().manual_seed(1)
    S, hkv, d, n = 3000, 8, 128, 777
    k_new = (3 * torch.randn(n, hkv, d, generator=g)).to(torch.bfloat16)
    v_new = (3 * torch.randn(n, hkv, d, generator=g)).to(torch.bfloat16)
    k_new[0, 0, :4] = torch.tensor([1e4, -1e4, 1e-7, 0.0]).to(torch.bfloat16)  # saturation, tiny
    ks = (0.01 + torch.rand(hkv, generator=g)).float()
    vs = (0.01 + torch.rand(hkv, generator=g)).float()
    slots = torch.randperm(S, generator=g)[:n].to(torch.int32)
    k8 = torch.zeros(S, hkv, d, dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    sa.seg_attn_kv_append_fp8(k_new.cuda(), v_new.cuda(), slots.cuda(), ks.cuda(), vs.cuda(), k8, v8)
    torch.cuda.synchronize()
    ek = (k_new.float() / ks.view(1, -1, 1)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    ev = (v_new.float() / vs.view(1, -1, 1)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(k8.cpu()[slots.long()], ek)
    assert torch.equal(v8.cpu()[slots.long()], ev)
    untouched = torch.ones(S, dtype=torch.bool)
    untouched[slots.long()] = False
    assert int(k8.cpu()[untouched].sum()) == 0
    assert sa.seg_attn_take_device_error() == 0


def _fp8_case(case):
    k8, v8, ks, vs = synth.fp8_pools(case["k_pool"], case["v_pool"])
    return dict(case, k8=k8, v8=v8, ks=ks, vs=vs)


def _run_fp8(case):
    q = case["q"].cuda()
    hq, d = q.shape[1], q.shape[2]
    tab = sa.SegTable.build(None, case["seg_starts"], case["seg_lens"], case["num_slots"], True,
                            sa.MODE_DECODE, hq, case["k8"].shape[1], d).to("cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device="cuda")
          if tab.workspace_bytes else None)
    sa.seg_attn_decode_fp8(q, case["k8"].cuda(), case["v8"].cuda(), case["ks"].cuda(),
                           case["vs"].cuda(), out, lse, tab.device, tab.desc, case["scale"], ws)
    torch.cuda.synchronize()
    return out, lse, tab


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 1), (16, 4), (4, 2), (8, 8)])
def test_fp8_decode_random(d, hq, hkv):
    case = _fp8_case(random_case(300 + d + hq + hkv, batch=5, hq=hq, hkv=hkv, d=d, causal=True,
                                 max_k=4000, nseg_max=6, q_mode="decode"))
    out, lse, _ = _run_fp8(case)
    ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                        case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                        case["scale"], True)
    compare(out, lse, ref_o, ref_l, f"fp8 decode d{d} {hq}/{hkv}")


def test_fp8_decode_multichunk_zero_and_tiny_segments():
    case = random_case(310, batch=6, hq=64, hkv=8, d=128, causal=True, max_k=9000, nseg_max=8,
                       q_mode="decode")
    case["seg_starts"][2], case["seg_lens"][2] = [], []
    g = torch.Generator().manual_seed(2)
    s3, l3 = [], []
    for s0, l0 in zip(case["seg_starts"][3], case["seg_lens"][3]):
        pos = s0
        while pos < s0 + l0:
            step = min(int(torch.randint(1, 4, (1,), generator=g)), s0 + l0 - pos)
            s3.append(pos)
            l3.append(step)
            pos += step
    case["seg_starts"][3], case["seg_lens"][3] = s3, l3
    case = _fp8_case(case)
    out, lse, tab = _run_fp8(case)
    assert tab.workspace_bytes > 0
    assert torch.all(out[2] == 0) and torch.all(torch.isneginf(lse[2]))
    ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                        case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                        case["scale"], True)
    compare(out, lse, ref_o, ref_l, "fp8 mixed")


def test_fp8_config4_sampled_requests():
    wl = synth.make_workload(4, device="cuda")
    b = wl.batches[0]
    k8, v8, ks, vs = synth.fp8_pools(wl.k_pool, wl.v_pool)
    tab = sa.SegTable.build(None, b.seg_starts, b.seg_lens, wl.num_slots, True, sa.MODE_DECODE,
                            wl.q_heads, wl.kv_heads, wl.head_dim).to("cuda")
    out = torch.empty_like(b.q)
    lse = torch.empty(b.q.shape[:2], dtype=torch.float32, device="cuda")
    ws = torch.empty(tab.workspace_bytes, dtype=torch.uint8, device="cuda")
    sa.seg_attn_decode_fp8(b.q, k8, v8, ks, vs, out, lse, tab.device, tab.desc, wl.scale, ws)
    torch.cuda.synchronize()
    reqs = [0, 17, 63, 127]
    wl8 = synth.Workload(config=4, name="", q_heads=wl.q_heads, kv_heads=wl.kv_heads,
                         head_dim=wl.head_dim, num_slots=wl.num_slots, scale=wl.scale,
                         batches=[b], k_pool=k8, v_pool=v8)
    sub = compact_requests(wl8, b, reqs)
    ref_o, ref_l = oracle.attention_fp8(sub["q_lens"], sub["seg_starts"], sub["seg_lens"],
                                        sub["q"], sub["k_pool"], sub["v_pool"], ks.cpu(),
                                        vs.cpu(), wl.scale, True)
    rows = sub["q_rows"].cuda()
    compare(out[rows], lse[rows], ref_o, ref_l, "fp8 config 4")
    assert sa.seg_attn_take_device_error() == 0


# ----------------------------------------------------------------- prefill over the FP8 cache
def _run_fp8_prefill(case):
    q = case["q"].cuda()
    hq, d = q.shape[1], q.shape[2]
    tab = sa.SegTable.build(case["q_lens"], case["seg_starts"], case["seg_lens"],
                            case["num_slots"], case["causal"], sa.MODE_PREFILL, hq,
                            case["k8"].shape[1], d).to("cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device="cuda")
          if tab.workspace_bytes else None)
    sa.seg_attn_prefill_fp8(q, case["k8"].cuda(), case["v8"].cuda(), case["ks"].cuda(),
                            case["vs"].cuda(), out, lse, tab.device, tab.desc, case["scale"], ws)
    torch.cuda.synchronize()
    return out, lse, tab


def _check_fp8_prefill(case, what):
    out, lse, tab = _run_fp8_prefill(case)
    ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                        case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                        case["scale"], case["causal"])
    compare(out, lse, ref_o, ref_l, what)
    return tab


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 1), (16, 4), (64, 8), (8, 8)])
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_prefill_random(d, hq, hkv, causal):
    # chunked prefill over prior context, ragged chunks and segments, several tiles
    case = _fp8_case(random_case(400 + d + hq + hkv + causal, batch=4, hq=hq, hkv=hkv, d=d,
                                 causal=causal, max_k=1500, nseg_max=5))
    _check_fp8_prefill(case, f"fp8 prefill d{d} {hq}/{hkv} causal={causal}")


def test_fp8_prefill_full_causal_and_tiny_segments():
    # whole-sequence causal prefill; one request cut into 1-3 slot runs so most tiles
    # are row-gathered rather than loaded as one box
    case = random_case(411, batch=3, hq=16, hkv=2, d=128, causal=True, max_k=700, q_mode="full")
    g = torch.Generator().manual_seed(3)
    s1, l1 = [], []
    for s0, l0 in zip(case["seg_starts"][1], case["seg_lens"][1]):
        pos = s0
        while pos < s0 + l0:
            step = min(int(torch.randint(1, 4, (1,), generator=g)), s0 + l0 - pos)
            s1.append(pos)
            l1.append(step)
            pos += step
    case["seg_starts"][1], case["seg_lens"][1] = s1, l1
    _check_fp8_prefill(_fp8_case(case), "fp8 full causal, tiny segments")


@pytest.mark.parametrize("causal", [True, False])
def test_fp8_prefill_split_items_merge(causal):
    # a few query tiles over a long context: items split along their keys, pieces merged
    g = torch.Generator().manual_seed(41)
    k_len, q_len, hq, hkv, d = 20000, 64, 16, 2, 128
    seg_lens = synth.split_uniform_cuts(k_len, 5, g)
    S = k_len + 300
    starts = synth.place_segments(seg_lens, S, g)
    k = torch.full((S, hkv, d), float("nan")).to(torch.bfloat16)
    v = k.clone()
    for s0, l in zip(starts, seg_lens):
        k[s0:s0 + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
        v[s0:s0 + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
    case = _fp8_case(dict(q=torch.randn(q_len, hq, d, generator=g).to(torch.bfloat16), k_pool=k,
                          v_pool=v, q_lens=[q_len], seg_starts=[starts], seg_lens=[seg_lens],
                          num_slots=S, scale=d ** -0.5, causal=causal))
    tab = _check_fp8_prefill(case, "fp8 split items")
    assert tab.desc.num_merge > 0


def test_fp8_prefill_short_chunks_one_tile_items():
    # chunks of at most 16 queries at G = 8: every item holds queries in its first
    # query tile only, so the one-tile kernel runs
    g = torch.Generator().manual_seed(43)
    case = random_case(413, batch=6, hq=64, hkv=8, d=128, causal=True, max_k=3000)
    case["q_lens"] = [int(torch.randint(1, 17, (1,), generator=g)) for _ in case["q_lens"]]
    case["q"] = torch.randn(sum(case["q_lens"]), 64, 128, generator=g).to(torch.bfloat16)
    tab = _check_fp8_prefill(_fp8_case(case), "fp8 short chunks")
    assert tab.desc.num_single == tab.desc.num_work


def test_fp8_prefill_zero_keys_and_empty_requests():
    case = random_case(414, batch=4, hq=8, hkv=2, d=64, causal=False, max_k=300)
    case["seg_starts"][1], case["seg_lens"][1] = [], []  # no keys: O = 0, lse = -inf
    case["q_lens"][2] = 0
    g = torch.Generator().manual_seed(44)
    case["q"] = torch.randn(sum(case["q_lens"]), 8, 64, generator=g).to(torch.bfloat16)
    _check_fp8_prefill(_fp8_case(case), "fp8 zero keys / empty request")


def test_fp8_prefill_large_scores_trigger_rescale():
    case = random_case(415, batch=2, hq=8, hkv=1, d=128, causal=True, max_k=800, q_mode="full")
    case["scale"] = 0.5
    _check_fp8_prefill(_fp8_case(case), "fp8 rescale")


def test_fp8_prefill_config5_sampled_rows():
    wl = synth.make_workload(5, device="cuda")
    b = wl.batches[1]
    k8, v8, ks, vs = synth.fp8_pools(wl.k_pool, wl.v_pool)
    tab = sa.SegTable.build(b.q_lens, b.seg_starts, b.seg_lens, wl.num_slots, True,
                            sa.MODE_PREFILL, wl.q_heads, wl.kv_heads, wl.head_dim).to("cuda")
    out = torch.empty_like(b.q)
    lse = torch.empty(b.q.shape[:2], dtype=torch.float32, device="cuda")
    ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device="cuda")
          if tab.workspace_bytes else None)
    sa.seg_attn_prefill_fp8(b.q, k8, v8, ks, vs, out, lse, tab.device, tab.desc, wl.scale, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    wl8 = synth.Workload(config=5, name="", q_heads=wl.q_heads, kv_heads=wl.kv_heads,
                         head_dim=wl.head_dim, num_slots=wl.num_slots, scale=wl.scale,
                         batches=[b], k_pool=k8, v_pool=v8)
    sub = compact_requests(wl8, b, [0])
    g = torch.Generator().manual_seed(6)
    toks = torch.cat([torch.tensor([0, 2047]), torch.randint(0, 2048, (14,), generator=g)])
    heads = torch.randint(0, wl.q_heads, (toks.numel(),), generator=g)
    ref_o, ref_l = oracle.attention_fp8(sub["q_lens"], sub["seg_starts"], sub["seg_lens"],
                                        sub["q"], sub["k_pool"], sub["v_pool"], ks.cpu(),
                                        vs.cpu(), wl.scale, True, rows=(toks.numpy(), heads.numpy()))
    compare(out[toks.cuda(), heads.cuda()], lse[toks.cuda(), heads.cuda()], ref_o, ref_l,
            "fp8 config 5 prefill")
    assert sa.seg_attn_take_device_error() == 0


@pytest.mark.parametrize("boost", [12.0, 100.0])
def test_fp8_prefill_late_score_jump(boost):
    # as the bf16 case: the reference max moves mid-row; P is f16 here, so a tile
    # whose scores jump by more than 2^15 must be redone from its own max
    case = random_case(417, batch=1, hq=8, hkv=1, d=128, causal=True, max_k=1200, q_mode="full")
    g = torch.Generator().manual_seed(29)
    u = torch.randn(128, generator=g)
    u = u / u.norm()
    case["q"] = (case["q"].float() + 3.0 * u).to(torch.bfloat16)
    k_len = sum(case["seg_lens"][0])
    slots = slots_of(case["seg_starts"][0], case["seg_lens"][0])
    for j in (k_len // 2, (3 * k_len) // 4):
        case["k_pool"][slots[j], 0] = (boost * u).to(torch.bfloat16)
    _check_fp8_prefill(_fp8_case(case), f"fp8 late score jump x{boost}")


# ----------------------------------------------------------------- shared prefixes, FP8 cache
def _run_fp8_any(case, decode, share):
    q = case["q"].cuda()
    hq, d = q.shape[1], q.shape[2]
    mode = (sa.MODE_DECODE if decode else sa.MODE_PREFILL) | (sa.SHARE_PREFIX if share else 0)
    tab = sa.SegTable.build(None if decode else case["q_lens"], case["seg_starts"],
                            case["seg_lens"], case["num_slots"], True, mode, hq,
                            case["k8"].shape[1], d).to("cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    ws = (torch.empty(tab.workspace_bytes, dtype=torch.uint8, device="cuda")
          if tab.workspace_bytes else None)
    fn = sa.seg_attn_decode_fp8 if decode else sa.seg_attn_prefill_fp8
    fn(q, case["k8"].cuda(), case["v8"].cuda(), case["ks"].cuda(), case["vs"].cuda(), out, lse,
       tab.device, tab.desc, case["scale"], ws)
    torch.cuda.synchronize()
    assert sa.seg_attn_take_device_error() == 0
    return out, lse, tab


def _check_fp8_shared(case, decode, what):
    out, lse, tab = _run_fp8_any(case, decode, True)
    assert tab.desc.shared == 1, what
    ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                        case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                        case["scale"], True)
    compare(out, lse, ref_o, ref_l, what)
    # every row against the unshared FP8 path (same products, other partial sums)
    out_u, lse_u, _ = _run_fp8_any(case, decode, False)
    assert (out.float() - out_u.float()).abs().max() <= 2 ** -7, what
    fin = torch.isfinite(lse_u)
    assert torch.equal(torch.isfinite(lse), fin), what
    assert (lse[fin] - lse_u[fin]).abs().max() <= 1e-4, what
    return tab


@pytest.mark.parametrize("seed", [0, 4])
@pytest.mark.parametrize("decode", [True, False])
def test_fp8_shared_prefix_random(seed, decode):
    reqs, q, S = shared_case(seed, B=8, decode=decode, max_prefix=5000)
    case = _fp8_case(shared_values(reqs, q, S, 64, 8, 128, seed=seed + 17))
    _check_fp8_shared(case, decode, f"fp8 shared {'decode' if decode else 'prefill'} s{seed}")


def test_fp8_shared_decode_group_wider_than_one_item():
    # 40 members x 8 heads = 320 packed rows: the prefix pass has two 256-row items
    rnd = np.random.default_rng(1)
    prefix = 5000
    pre = [(0, prefix // 3), (prefix // 3 + 50, prefix - prefix // 3)]
    nxt = prefix + 100
    reqs = []
    for _ in range(40):
        own = int(rnd.integers(1, 701))
        reqs.append(([s for s, _ in pre] + [nxt], [l for _, l in pre] + [own]))
        nxt += own + int(rnd.integers(0, 9))
    case = _fp8_case(shared_values(reqs, [1] * 40, nxt + 10, 64, 8, 128, seed=3))
    tab = _check_fp8_shared(case, True, "fp8 shared decode, 40 members")
    assert tab.desc.num_group_work > 2 * tab.desc.kv_heads
