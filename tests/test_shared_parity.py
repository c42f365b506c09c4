"""GPU parity of the shared-prefix path (SEG_ATTN_SHARE_PREFIX) against the fp64 oracle.

The oracle computes each request on its own (shared slots are simply read by
every request that lists them), so sharing must not change any result beyond
fp32 rounding.  Covers decode and causal / non-causal prefill, prefix passes
split into several pieces, groups wider than one 256-row item, empty own key
ranges, members without queries, and the full-size shared-prefix configs
(sampled rows against the oracle, every row against the unshared path)."""
import math

import numpy as np
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import synth

from helpers import compare, run_cuda, shared_case, shared_values

pytestmark = pytest.mark.gpu


def _run(case, decode, share=True, causal=True):
    c = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    mode = (sa.MODE_DECODE if decode else sa.MODE_PREFILL) | (sa.SHARE_PREFIX if share else 0)
    out, lse, tab = run_cuda(c["q"], c["k_pool"], c["v_pool"], None if decode else c["q_lens"],
                             c["seg_starts"], c["seg_lens"], c["num_slots"], causal, mode,
                             c["scale"])
    torch.cuda.synchronize()
    assert sa.seg_attn_take_device_error() == 0
    return out, lse, tab


def _check(case, decode, what, causal=True, want_shared=True):
    out, lse, tab = _run(case, decode, causal=causal)
    if want_shared:
        assert tab.desc.shared == 1, what
    ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                    case["q"], case["k_pool"], case["v_pool"], case["scale"],
                                    causal)
    return compare(out, lse, ref_o, ref_l, what), tab


@pytest.mark.parametrize("seed", [0, 3, 4, 5])
@pytest.mark.parametrize("decode", [True, False])
@pytest.mark.parametrize("d,hq,hkv", [(128, 64, 8), (64, 16, 2), (128, 8, 8)])
def test_shared_random(seed, decode, d, hq, hkv):
    reqs, q, S = shared_case(seed, B=8, decode=decode, max_prefix=5000)
    case = shared_values(reqs, q, S, hq, hkv, d, seed=seed + 17)
    _check(case, decode, f"shared {'decode' if decode else 'prefill'} s{seed} d{d} {hq}/{hkv}")


def _group_case(members, prefix, own_max, seed, decode, hq=64, hkv=8, d=128, q_max=24):
    rnd = np.random.default_rng(seed)
    pre = [(0, prefix // 3), (prefix // 3 + 50, prefix - prefix // 3)]  # two prefix segments
    nxt = prefix + 100
    reqs, q = [], []
    for _ in range(members):
        own = int(rnd.integers(1, own_max + 1))
        reqs.append(([s for s, _ in pre] + [nxt], [l for _, l in pre] + [own]))
        nxt += own + int(rnd.integers(0, 9))
        q.append(1 if decode else int(rnd.integers(1, min(q_max, own) + 1)))
    return shared_values(reqs, q, nxt + 10, hq, hkv, d, seed)


def test_decode_group_wider_than_one_item_and_split_prefix_pass():
    # 40 members x 8 heads = 320 packed rows: two 256-row items over a 5000-key prefix
    case = _group_case(40, 5000, 700, seed=1, decode=True)
    _, tab = _check(case, True, "decode 40 members")
    d = tab.desc
    gw = tab.host[d.off_group_work: d.off_group_work + 16 * d.num_group_work].view(-1, 16)
    assert set(gw[:, 2].tolist()) == {0, 32}           # two query blocks
    assert d.num_group_work > 2 * d.kv_heads            # pieces along the prefix


def test_prefill_group_packs_short_chunks():
    case = _group_case(12, 3000, 200, seed=2, decode=False)
    _check(case, False, "prefill 12 members")


def test_empty_own_keys_and_identical_requests():
    # request 0 == request 1; request 2 extends them by 30 keys: only it has own keys
    reqs = [([0, 1000], [700, 300]), ([0, 1000], [700, 300]), ([0, 1000, 2000], [700, 300, 30])]
    case = shared_values(reqs, [1, 1, 1], 2100, 32, 4, 128, seed=3)
    _, tab = _check(case, True, "decode identical")
    assert tab.host[tab.desc.off_k_lens: tab.desc.off_k_lens + 3].tolist() == [0, 0, 30]


def test_prefill_member_without_queries_and_non_causal():
    reqs = [([0, 3000], [2000, 40]), ([0, 3100], [2000, 60]), ([0, 3200], [2000, 35])]
    case = shared_values(reqs, [10, 0, 20], 3300, 16, 2, 64, seed=4)
    _check(case, False, "prefill q=0 member")
    _check(case, False, "prefill non-causal", causal=False)


def test_mixed_shared_and_unshared_decode_requests():
    # a sharing pair, a long loner (several chunks) and a short loner (one chunk)
    reqs = [([0, 5000], [3000, 100]), ([0, 5200], [3000, 90]), ([6000], [9000]),
            ([16000], [50])]
    case = shared_values(reqs, [1] * 4, 16100, 64, 8, 128, seed=5)
    _, tab = _check(case, True, "decode mixed")
    d = tab.desc
    casc = tab.host[d.off_cascade: d.off_cascade + 8 * d.num_cascade].view(-1, 8)
    assert casc[:, 0].tolist() == [0, 1, 2]  # the short loner writes its own result


def _sample_rows(n_rows, hq, count, seed):
    rnd = np.random.default_rng(seed)
    tok = np.concatenate([[0, n_rows - 1], rnd.integers(0, n_rows, count - 2)]).astype(np.int64)
    head = rnd.integers(0, hq, count).astype(np.int32)
    return tok, head


@pytest.mark.parametrize("cfg", [6, 7])
def test_shared_prefix_config_full_size(cfg):
    wl = synth.make_workload(cfg, device="cuda")
    b = wl.batches[0]
    decode = b.mode == "decode"
    mode = sa.MODE_DECODE if decode else sa.MODE_PREFILL
    args = (b.q, wl.k_pool, wl.v_pool, None if decode else b.q_lens, b.seg_starts, b.seg_lens,
            wl.num_slots, True)
    out_s, lse_s, tab = run_cuda(*args, mode | sa.SHARE_PREFIX, wl.scale)
    out_p, lse_p, _ = run_cuda(*args, mode, wl.scale)
    torch.cuda.synchronize()
    assert tab.desc.shared == 1 and sa.seg_attn_take_device_error() == 0
    # every row: the shared path agrees with the unshared one to bf16 output rounding
    diff = (out_s.float() - out_p.float()).abs()
    assert torch.isfinite(out_s).all() and float(diff.max()) <= 2e-2
    assert float(diff.mean()) <= 1e-3
    assert float(((lse_s - lse_p).abs() / lse_p.abs().clamp(min=1)).max()) <= 1e-4
    # sampled rows against the oracle
    tok, head = _sample_rows(b.total_q, wl.q_heads, 96, seed=cfg)
    ref_o, ref_l = oracle.attention(b.q_lens, b.seg_starts, b.seg_lens, b.q.cpu(),
                                    wl.k_pool.cpu(), wl.v_pool.cpu(), wl.scale, True,
                                    rows=(tok, head))
    t, h = torch.from_numpy(tok).cuda(), torch.from_numpy(head).long().cuda()
    compare(out_s[t, h], lse_s[t, h], ref_o, ref_l, f"config {cfg} shared")
