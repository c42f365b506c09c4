"""KV append kernel (bit-exact scatter) and an allocator-driven serving loop whose
attention results are checked against the oracle after every step."""
import math

import numpy as np
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa

from helpers import compare, run_cuda

pytestmark = pytest.mark.gpu


def test_append_is_a_bit_exact_scatter():
    g = torch.Generator().manual_seed(0)
    S, hkv, d, n = 5000, 8, 128, 1234
    k_pool = torch.randn(S, hkv, d, generator=g).to(torch.bfloat16)
    v_pool = torch.randn(S, hkv, d, generator=g).to(torch.bfloat16)
    slots = torch.randperm(S, generator=g)[:n].to(torch.int32)
    k_new = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16)
    v_new = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16)
    kd, vd = k_pool.cuda(), v_pool.cuda()
    sa.seg_attn_kv_append(k_new.cuda(), v_new.cuda(), slots.cuda(), kd, vd)
    torch.cuda.synchronize()
    ke, ve = k_pool.clone(), v_pool.clone()
    ke[slots.long()] = k_new
    ve[slots.long()] = v_new
    assert torch.equal(kd.cpu().view(torch.int16), ke.view(torch.int16))
    assert torch.equal(vd.cpu().view(torch.int16), ve.view(torch.int16))
    assert sa.seg_attn_take_device_error() == 0


def test_append_skips_and_flags_out_of_range_slots():
    S, hkv, d = 64, 2, 64
    k_pool = torch.zeros(S, hkv, d, dtype=torch.bfloat16, device="cuda")
    v_pool = torch.zeros_like(k_pool)
    slots = torch.tensor([3, -1, 64, 10], dtype=torch.int32, device="cuda")
    new = torch.ones(4, hkv, d, dtype=torch.bfloat16, device="cuda")
    sa.seg_attn_kv_append(new, new, slots, k_pool, v_pool)
    torch.cuda.synchronize()
    assert sa.seg_attn_take_device_error() == 2
    assert sa.seg_attn_take_device_error() == 0
    written = (k_pool.float().abs().sum(dim=(1, 2)) > 0).nonzero().flatten().tolist()
    assert written == [3, 10]


def test_serving_loop_allocator_append_attention():
    """Chunked prefills and decodes of several sequences through the allocator; every
    step appends the new tokens' K/V, rebuilds the table from the allocator's segment
    lists and checks attention against the oracle on a host copy of the pools."""
    g = torch.Generator().manual_seed(11)
    S, hq, hkv, d = 6000, 16, 4, 128
    scale = 1 / math.sqrt(d)
    pool = sa.SegPool(S)
    k_pool = torch.full((S, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_pool = torch.full_like(k_pool, float("nan"))
    lens = {}

    def add_tokens(seq, n):
        slots = torch.from_numpy(pool.append(seq, n)).cuda()
        kn = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16).cuda()
        vn = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16).cuda()
        sa.seg_attn_kv_append(kn, vn, slots, k_pool, v_pool)
        lens[seq] = lens.get(seq, 0) + n

    def check(seqs, q_lens, mode):
        segs = [pool.segments(s) for s in seqs]
        q = torch.randn(sum(q_lens), hq, d, generator=g).to(torch.bfloat16)
        out, lse, _ = run_cuda(q.cuda(), k_pool, v_pool, q_lens if mode == sa.MODE_PREFILL else None,
                               [s for s, _ in segs], [l for _, l in segs], S, True, mode, scale)
        torch.cuda.synchronize()
        ref_o, ref_l = oracle.attention(q_lens, [s for s, _ in segs], [l for _, l in segs], q,
                                        k_pool.cpu(), v_pool.cpu(), scale, True)
        compare(out, lse, ref_o, ref_l, f"{mode} {seqs}")
        return max(len(s) for s, _ in segs)

    # prefill three sequences in chunks (each chunk's K/V appended before its attention)
    for chunk in ([300, 500, 200], [100, 40, 257]):
        for seq, n in zip((1, 2, 3), chunk):
            add_tokens(seq, n)
        check([1, 2, 3], list(chunk), sa.MODE_PREFILL)
    # decode steps
    for _ in range(3):
        for seq in (1, 2, 3):
            add_tokens(seq, 1)
        check([1, 2, 3], [1, 1, 1], sa.MODE_DECODE)
    # free the middle sequence, start a long one that must reuse the hole -> several segments
    pool.release(2)
    add_tokens(4, 2500)
    max_segs = check([1, 3, 4], [1, 1, 5], sa.MODE_PREFILL)
    assert max_segs >= 2
    for _ in range(2):
        for seq in (1, 3, 4):
            add_tokens(seq, 1)
        check([1, 3, 4], [1, 1, 1], sa.MODE_DECODE)
    assert pool.stats()["free_slots"] == S - sum(v for k, v in lens.items() if k != 2)
    assert sa.seg_attn_take_device_error() == 0
