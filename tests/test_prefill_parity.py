"""GPU parity of seg_attn_prefill (tcgen05 / TMEM / TMA gather) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import synth

from helpers import compact_requests, compare, random_case, run_batch, run_cuda, slots_of

pytestmark = pytest.mark.gpu


def _run(case, causal=None):
    causal = case["causal"] if causal is None else causal
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    out, lse, tab = run_cuda(dev["q"], dev["k_pool"], dev["v_pool"], case["q_lens"],
                             case["seg_starts"], case["seg_lens"], case["num_slots"], causal,
                             sa.MODE_PREFILL, case["scale"])
    torch.cuda.synchronize()
    return out, lse, tab


def _check(case, what):
    out, lse, tab = _run(case)
    ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                    case["q"], case["k_pool"], case["v_pool"], case["scale"],
                                    case["causal"])
    return compare(out, lse, ref_o, ref_l, what)


def test_config1_tiny():
    wl = synth.make_workload(1)
    b = wl.batches[0]
    case = dict(q=b.q, k_pool=wl.k_pool, v_pool=wl.v_pool, q_lens=b.q_lens,
                seg_starts=b.seg_starts, seg_lens=b.seg_lens, num_slots=wl.num_slots,
                scale=wl.scale, causal=b.causal)
    _check(case, "config 1")


def test_config2_pages_shaped_full():
    wl = synth.make_workload(2)
    b = wl.batches[0]
    case = dict(q=b.q, k_pool=wl.k_pool, v_pool=wl.v_pool, q_lens=b.q_lens,
                seg_starts=b.seg_starts, seg_lens=b.seg_lens, num_slots=wl.num_slots,
                scale=wl.scale, causal=b.causal)
    _check(case, "config 2")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 1), (8, 2), (4, 4), (32, 2)])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_random(d, hq, hkv, causal):
    case = random_case(1000 + d + 7 * hq + hkv + causal, batch=4, hq=hq, hkv=hkv, d=d,
                       causal=causal, max_k=700, nseg_max=5, q_mode="chunk")
    _check(case, f"prefill d{d} {hq}/{hkv} causal={causal}")


def test_prefill_full_causal_many_tiles():
    # q = k (no prior context): diagonal masking on every tile of both query tiles
    case = random_case(21, batch=3, hq=16, hkv=2, d=128, causal=True, max_k=900, nseg_max=3,
                       q_mode="full")
    _check(case, "full causal")


def test_prefill_tiny_segments_gather():
    # 1..3-slot segments: every gathered row comes from a different run
    case = random_case(22, batch=2, hq=8, hkv=1, d=128, causal=True, max_k=400, nseg_max=1)
    g = torch.Generator().manual_seed(4)
    new_s, new_l = [], []
    for ss, ll in zip(case["seg_starts"], case["seg_lens"]):
        s2, l2 = [], []
        for s, l in zip(ss, ll):
            pos = s
            while pos < s + l:
                step = min(int(torch.randint(1, 4, (1,), generator=g)), s + l - pos)
                s2.append(pos)
                l2.append(step)
                pos += step
        new_s.append(s2)
        new_l.append(l2)
    case["seg_starts"], case["seg_lens"] = new_s, new_l
    _check(case, "tiny segments")


def test_prefill_zero_keys_noncausal_and_zero_queries():
    case = random_case(23, batch=3, hq=8, hkv=2, d=128, causal=False, max_k=300)
    case["q_lens"] = [3, 0, 2]
    case["q"] = case["q"][:5] if case["q"].shape[0] >= 5 else torch.randn(5, 8, 128).to(torch.bfloat16)
    case["seg_starts"][2], case["seg_lens"][2] = [], []
    out, lse, _ = _run(case)
    assert torch.all(out[3:] == 0) and torch.all(torch.isneginf(lse[3:]))
    ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                    case["q"], case["k_pool"], case["v_pool"], case["scale"], False)
    compare(out, lse, ref_o, ref_l, "zero keys")


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_split_items_merge(causal):
    # few query tiles over a long context: the planner splits items along their keys,
    # the pieces' partials are merged by the second kernel
    g = torch.Generator().manual_seed(31)
    k_len, q_len, hq, hkv, d = 20000, 64, 16, 2, 128
    seg_lens = synth.split_uniform_cuts(k_len, 5, g)
    S = k_len + 300
    starts = synth.place_segments(seg_lens, S, g)
    k = torch.full((S, hkv, d), float("nan")).to(torch.bfloat16)
    v = k.clone()
    for s0, l in zip(starts, seg_lens):
        k[s0:s0 + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
        v[s0:s0 + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
    case = dict(q=torch.randn(q_len, hq, d, generator=g).to(torch.bfloat16), k_pool=k, v_pool=v,
                q_lens=[q_len], seg_starts=[starts], seg_lens=[seg_lens], num_slots=S,
                scale=d ** -0.5, causal=causal)
    out, lse, tab = _run(case)
    assert tab.desc.num_merge > 0
    ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                    case["q"], k, v, case["scale"], causal)
    compare(out, lse, ref_o, ref_l, "split items")


def test_prefill_large_scores_trigger_rescale():
    # scaled-up queries make the running max jump by more than 2^8 across tiles
    case = random_case(24, batch=2, hq=8, hkv=1, d=128, causal=True, max_k=800, q_mode="full")
    case["scale"] = 0.5
    _check(case, "rescale")


@pytest.mark.parametrize("boost", [12.0, 25.0, 100.0])
def test_prefill_late_score_jump(boost):
    # one key deep in the context aligned with a direction every query leans on: its
    # score jumps past all earlier ones by a few to many powers of two, so the
    # reference max moves mid-row (deferred to the next tile, or the tile is redone)
    case = random_case(27, batch=1, hq=8, hkv=1, d=128, causal=True, max_k=1200, q_mode="full")
    g = torch.Generator().manual_seed(28)
    u = torch.randn(128, generator=g)
    u = u / u.norm()
    q = case["q"].float() + 3.0 * u
    case["q"] = q.to(torch.bfloat16)
    k_len = sum(case["seg_lens"][0])
    slots = slots_of(case["seg_starts"][0], case["seg_lens"][0])
    for j in (k_len // 2, (3 * k_len) // 4):
        case["k_pool"][slots[j], 0] = (boost * u).to(torch.bfloat16)
    _check(case, f"late score jump x{boost}")


@pytest.mark.parametrize("d,hq,hkv,q_max", [(128, 64, 8, 16), (64, 16, 4, 32), (128, 8, 8, 128)])
def test_prefill_short_chunks_run_the_one_tile_kernel(d, hq, hkv, q_max):
    # every request's chunk fits one 128-row query tile, so the whole pass runs the
    # one-tile kernel (double-buffered S, three-stage K/V ring); long prior contexts
    # give each item many K tiles through the ring, some of them gathered
    g = torch.Generator().manual_seed(47 + d + hq)
    case = random_case(416 + d + hq, batch=6, hq=hq, hkv=hkv, d=d, causal=True, max_k=5000,
                       nseg_max=6)
    # at most 128 / G queries per request (one query tile), never more than its keys
    case["q_lens"] = [min(sum(l), int(torch.randint(1, q_max + 1, (1,), generator=g)))
                      for l in case["seg_lens"]]
    case["q"] = torch.randn(sum(case["q_lens"]), hq, d, generator=g).to(torch.bfloat16)
    _, _, tab = _run(case)
    assert tab.desc.num_single == tab.desc.num_work > 0
    _check(case, f"one-tile kernel d{d} {hq}/{hkv}")


def test_decode_row_equals_last_prefill_row():
    case = random_case(25, batch=2, hq=8, hkv=1, d=128, causal=True, max_k=600, q_mode="full")
    out, lse, _ = _run(case)
    last = np.cumsum(case["q_lens"]) - 1
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    out_d, lse_d, _ = run_cuda(dev["q"][torch.tensor(last).cuda()], dev["k_pool"], dev["v_pool"],
                               None, case["seg_starts"], case["seg_lens"], case["num_slots"], True,
                               sa.MODE_DECODE, case["scale"])
    torch.cuda.synchronize()
    assert (out_d.float() - out[last].float()).abs().max() <= 2 ** -7
    assert (lse_d - lse[last]).abs().max() <= 1e-4


def test_config3_all_requests():
    # every row of all 16 requests of the chunked varlen batch (about 2.8e11 flop in the
    # oracle), in the launch configuration the benchmark times
    wl = synth.make_workload(3, device="cuda")
    b = wl.batches[0]
    out, lse, _ = run_batch(wl, b)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    reqs = [r for r in range(b.batch) if b.q_lens[r] > 0]
    assert sum(b.q_lens[r] for r in reqs) == b.total_q
    sub = compact_requests(wl, b, reqs)
    ref_o, ref_l = oracle.attention(sub["q_lens"], sub["seg_starts"], sub["seg_lens"], sub["q"],
                                    sub["k_pool"], sub["v_pool"], wl.scale, True)
    rows = sub["q_rows"].cuda()
    compare(out[rows], lse[rows], ref_o, ref_l, "config 3")


def config5_prefill_rows(qpt, span, q_len, q_heads, kv_heads, seed=5):
    """(token, head) rows of the 2048-query chunk that reach every work item of the plan:
    for each 2-tile item (span queries) one query in each of its two query tiles and, for
    each kv head, one query head of its group; plus every head of the first and last
    query.  Each row attends to all key tiles, so every split piece of every item (first
    and last key tile included) contributes to some checked row."""
    g = torch.Generator().manual_seed(seed)
    group = q_heads // kv_heads
    toks, heads = [], []
    for q0 in range(0, q_len, span):
        for t in range(2):
            lo = q0 + t * qpt
            if lo >= q_len:
                continue
            for kv in range(kv_heads):
                toks.append(lo + int(torch.randint(0, min(qpt, q_len - lo), (1,), generator=g)))
                heads.append(kv * group + int(torch.randint(0, group, (1,), generator=g)))
    for tok in (0, q_len - 1):
        toks += [tok] * q_heads
        heads += list(range(q_heads))
    return torch.tensor(toks), torch.tensor(heads)


def test_config5_prefill_rows_of_every_item():
    wl = synth.make_workload(5, device="cuda")
    b = wl.batches[1]
    out, lse, tab = run_batch(wl, b)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert tab.desc.num_merge > 0  # the items are split along their keys at this size
    qpt = tab.desc.queries_per_tile
    toks, heads = config5_prefill_rows(qpt, 2 * qpt, b.q_lens[0], wl.q_heads, wl.kv_heads)
    assert toks.numel() >= 1024
    sub = compact_requests(wl, b, [0])
    ref_o, ref_l = oracle.attention(sub["q_lens"], sub["seg_starts"], sub["seg_lens"], sub["q"],
                                    sub["k_pool"], sub["v_pool"], wl.scale, True,
                                    rows=(toks.numpy(), heads.numpy()))
    compare(out[toks.cuda(), heads.cuda()], lse[toks.cuda(), heads.cuda()], ref_o, ref_l,
            "config 5 prefill")


def test_no_device_error_recorded():
    assert sa.seg_attn_take_device_error() == 0
