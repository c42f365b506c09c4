"""Shared-prefix plans (SEG_ATTN_SHARE_PREFIX) on the host, without a GPU.

Checks the builder's grouping against a brute-force model (every partition of
the batch into runs of consecutive requests), and the table it writes: each
request's keys split into its group's prefix and its own keys, the pass over
the prefixes, and the rows the cascade merge completes."""
import itertools
import math

import numpy as np
import pytest

import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import _build, synth

from helpers import shared_case, slots_of

MIN_SHARED = 256  # shortest prefix the builder shares
TILE = 128


@pytest.fixture(scope="module", autouse=True)
def built_library():
    _build.build()
    return sa.load_library()


def arr(tab, off, n, width=1):
    a = tab.host[off: off + n * width].numpy().copy()
    return a.reshape(-1, width) if width > 1 else a


def lcp(a, b):
    n = 0
    while n < min(len(a), len(b)) and a[n] == b[n]:
        n += 1
    return n


def model_best_saving(slot_lists, q_lens, cap, span):
    """Largest saving over every partition into consecutive groups (brute force)."""
    B = len(slot_lists)

    def saving(j, i):
        if i - j < 2:
            return 0
        P = min(cap[j:i])
        for r in range(j + 1, i):
            P = min(P, lcp(slot_lists[r - 1], slot_lists[r]))
        if P < MIN_SHARED:
            return None
        reads = lambda q: -(-q // span)
        s = (sum(reads(q) for q in q_lens[j:i]) - reads(sum(q_lens[j:i]))) * -(-P // TILE)
        return s if s > 0 else None

    best = 0
    for cuts in itertools.product([0, 1], repeat=max(0, B - 1)):
        ends = [i + 1 for i, c in enumerate(cuts) if c] + [B]
        total, j, ok = 0, 0, True
        for i in ends:
            s = saving(j, i)
            if s is None:
                ok = False
                break
            total += s
            j = i
        if ok:
            best = max(best, total)
    return best, saving


def build(reqs, q, num_slots, decode, share=True, causal=True, hq=16, hkv=2, d=128):
    mode = (sa.MODE_DECODE if decode else sa.MODE_PREFILL) | (sa.SHARE_PREFIX if share else 0)
    return sa.SegTable.build(None if decode else q, [s for s, _ in reqs], [l for _, l in reqs],
                             num_slots, causal, mode, hq, hkv, d)


def check_plan(tab, reqs, q, decode, causal=True, hq=16, hkv=2):
    d = tab.desc
    B = len(reqs)
    G = hq // hkv
    span = 2 * (128 // G)
    slot_lists = [slots_of(*r) for r in reqs]
    k = [len(s) for s in slot_lists]
    cap = [k[r] - q[r] if (causal and not decode) else k[r] for r in range(B)]
    best, saving = model_best_saving(slot_lists, q, cap, span)
    if d.shared == 0:
        assert best == 0
        return
    greq = arr(tab, d.off_group_req, d.num_groups + 1)
    P = arr(tab, d.off_group_k_lens, d.num_groups)
    assert greq[0] == 0 and greq[-1] == B and (np.diff(greq) > 0).all()
    # the plan's groups are valid and reach the model's best saving
    total = 0
    for p in range(d.num_groups):
        j, i = int(greq[p]), int(greq[p + 1])
        s = saving(j, i)
        assert s is not None, (j, i)
        total += s
        if i - j >= 2:
            want = min(cap[j:i] + [lcp(slot_lists[r - 1], slot_lists[r]) for r in range(j + 1, i)])
            assert P[p] == want
        else:
            assert P[p] == 0
    assert total == best
    # each request's keys = its group's prefix keys, then its own keys
    g_off = arr(tab, d.off_group_seg_offsets, d.num_groups + 1)
    g_start = arr(tab, d.off_group_seg_start, d.num_group_segments)
    g_len = arr(tab, d.off_group_seg_len, d.num_group_segments)
    g_kst = arr(tab, d.off_group_seg_kstart, d.num_group_segments)
    s_off = arr(tab, d.off_seg_offsets, B + 1)
    s_start = arr(tab, d.off_seg_start, d.num_segments)
    s_len = arr(tab, d.off_seg_len, d.num_segments)
    s_kst = arr(tab, d.off_seg_kstart, d.num_segments)
    k_lens = arr(tab, d.off_k_lens, B)
    gq = arr(tab, d.off_group_q_offsets, d.num_groups + 1)
    q_off = np.concatenate([[0], np.cumsum(q)])
    assert (gq == q_off[greq]).all()
    group_of = np.repeat(np.arange(d.num_groups), np.diff(greq))
    for r in range(B):
        p = group_of[r]
        a, b = g_off[p], g_off[p + 1]
        pre = slots_of(g_start[a:b], g_len[a:b])
        own = slots_of(s_start[s_off[r]:s_off[r + 1]], s_len[s_off[r]:s_off[r + 1]])
        assert len(pre) == P[p] and pre + own == slot_lists[r]
        assert k_lens[r] == k[r] - P[p]
        assert list(s_kst[s_off[r]:s_off[r + 1]]) == list(np.cumsum([0] + list(s_len[s_off[r]:s_off[r + 1]]))[:-1])
        assert list(g_kst[a:b]) == list(np.cumsum([0] + list(g_len[a:b]))[:-1])
    assert d.group_total_k == int(P.sum())
    # the prefix pass: every (group, query block, kv head) item covers its tiles once,
    # every piece writes a partial into its own slot
    gw = arr(tab, d.off_group_work, d.num_group_work, 16)
    cit = arr(tab, d.off_citem, d.num_citems, 4)
    used = set()
    for p in range(d.num_groups):
        gq_n = gq[p + 1] - gq[p]
        for q0 in range(0, gq_n if P[p] > 0 else 0, span):
            for g in range(hkv):
                pcs = gw[(gw[:, 0] == p) & (gw[:, 1] == g) & (gw[:, 2] == q0)]
                pcs = pcs[np.argsort(pcs[:, 3])]
                assert pcs[0, 3] == 0 and pcs[-1, 4] == math.ceil(P[p] / TILE)
                assert (pcs[1:, 3] == pcs[:-1, 4]).all() and (pcs[:, 5] >= 0).all()
                used |= set(pcs[:, 5].tolist())
    assert used == set(range(d.num_group_parts)) and len(gw) == d.num_group_parts
    # cascade rows
    casc = arr(tab, d.off_cascade, d.num_cascade, 8)
    if decode:
        rc = arr(tab, d.off_req_chunks, B + 1)
        want_rows = [r for r in range(B) if P[group_of[r]] > 0 or rc[r + 1] - rc[r] > 1]
        assert casc[:, 0].tolist() == want_rows and casc[:, 1].tolist() == want_rows
        work = arr(tab, d.off_work, d.num_work, 4)
        for r in range(B):
            shared_r = P[group_of[r]] > 0
            n = rc[r + 1] - rc[r]
            assert (work[rc[r]:rc[r + 1], 3] == (0 if shared_r else n)).all()
    else:
        want_rows = [int(q_off[r] + i) for r in range(B) if P[group_of[r]] > 0 for i in range(q[r])]
        assert casc[:, 0].tolist() == want_rows
    for row, r, pc, pl, sc, sl, _, _ in casc:
        p = group_of[r]
        if P[p] > 0:
            assert pl == row - gq[p]
            slot0, parts, q0, _ = cit[pc]
            assert q0 <= pl < q0 + span
            for g in range(hkv):  # the listed item is kv head 0; head g follows at +g
                assert cit[pc + g][2] == q0
        else:
            assert pc == -1
        if not decode:
            assert sl == row - q_off[r] and cit[sc][2] <= sl < cit[sc][2] + span


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("decode", [True, False])
def test_grouping_matches_brute_force_and_table_is_consistent(seed, decode):
    reqs, q, S = shared_case(seed, B=8, decode=decode)
    tab = build(reqs, q, S, decode)
    check_plan(tab, reqs, q, decode)


def test_sharing_is_seen_through_different_segment_cuts():
    # the same 600 slots, cut 1 / 2 / 3 ways, then each request's own keys
    reqs = [([1000, 5000], [600, 40]),
            ([1000, 1300, 6000], [300, 300, 50]),
            ([1000, 1100, 1350, 7000], [100, 250, 250, 60])]
    tab = build(reqs, [1, 1, 1], 8000, decode=True)
    d = tab.desc
    assert d.shared == 1 and d.num_groups == 1
    assert arr(tab, d.off_group_k_lens, 1).tolist() == [600]
    check_plan(tab, reqs, [1, 1, 1], True)


def test_identical_requests_and_a_request_that_is_a_prefix_of_another():
    reqs = [([0], [700]), ([0], [700]), ([0, 900], [700, 30])]
    tab = build(reqs, [1, 1, 1], 1000, decode=True)
    d = tab.desc
    assert d.shared == 1 and arr(tab, d.off_group_k_lens, d.num_groups).tolist() == [700]
    assert arr(tab, d.off_k_lens, 3).tolist() == [0, 0, 30]
    check_plan(tab, reqs, [1, 1, 1], True)


def test_causal_prefill_prefix_stops_before_new_tokens():
    # both requests' first 500 slots agree, but request 1 has 450 prior keys only
    reqs = [([0, 600], [500, 20]), ([0], [500])]
    q = [10, 50]
    tab = build(reqs, q, 700, decode=False)
    d = tab.desc
    assert d.shared == 1 and arr(tab, d.off_group_k_lens, 1).tolist() == [450]
    check_plan(tab, reqs, q, False)
    # without the causal mask every key is visible to every query: all 500 are shared
    tab = build(reqs, q, 700, decode=False, causal=False)
    assert arr(tab, tab.desc.off_group_k_lens, 1).tolist() == [500]


def test_no_common_prefix_gives_the_plain_table():
    reqs = [([0], [300]), ([400], [300]), ([800], [200])]
    for decode, q in ((True, [1, 1, 1]), (False, [5, 7, 9])):
        plain = build(reqs, q, 1100, decode, share=False)
        tab = build(reqs, q, 1100, decode, share=True)
        assert tab.desc.shared == 0
        assert bytes(tab.desc) == bytes(plain.desc)
        assert tab.host.equal(plain.host)


def test_short_prefixes_are_not_shared():
    reqs = [([0, 500], [255, 10]), ([0, 600], [255, 10])]
    tab = build(reqs, [1, 1], 700, decode=True)
    assert tab.desc.shared == 0


def test_unknown_mode_flags_are_rejected():
    with pytest.raises(sa.SegAttnError) as e:
        sa.SegTable.build(None, [[0]], [[10]], 20, True, sa.MODE_DECODE | 0x200, 16, 2, 128)
    assert e.value.code == sa.STATUS["INVALID_ARG"]


@pytest.mark.parametrize("cfg", [6, 7])
def test_shared_prefix_configs_share_every_group(cfg):
    wl = synth.make_workload(cfg, values=False)
    b = wl.batches[0]
    decode = b.mode == "decode"
    mode = (sa.MODE_DECODE if decode else sa.MODE_PREFILL) | sa.SHARE_PREFIX
    tab = sa.SegTable.build(None if decode else b.q_lens, b.seg_starts, b.seg_lens, wl.num_slots,
                            True, mode, wl.q_heads, wl.kv_heads, wl.head_dim)
    d = tab.desc
    assert d.shared == 1
    P = arr(tab, d.off_group_k_lens, d.num_groups)
    greq = arr(tab, d.off_group_req, d.num_groups + 1)
    members = 8
    if decode:
        # one group per generated group, its prefix exactly the generated one
        assert greq.tolist() == list(range(0, b.batch + 1, members))
        for p in range(d.num_groups):
            lists = [list(zip(b.seg_starts[r], b.seg_lens[r]))
                     for r in range(p * members, (p + 1) * members)]
            n = 0
            while all(len(x) > n and x[n] == lists[0][n] for x in lists):
                n += 1
            assert P[p] == sum(l for _, l in lists[0][:n])  # the generated prefix
    # fewer K tiles in total than the plain plan
    plain = sa.SegTable.build(None if decode else b.q_lens, b.seg_starts, b.seg_lens, wl.num_slots,
                              True, mode & 0xff, wl.q_heads, wl.kv_heads, wl.head_dim)
    if not decode:
        tiles = lambda t, off, n: int((arr(t, off, n, 16)[:, 4] - arr(t, off, n, 16)[:, 3]).sum())
        shared_tiles = tiles(tab, d.off_work, d.num_work) + tiles(tab, d.off_group_work,
                                                                  d.num_group_work)
        assert shared_tiles < 0.8 * tiles(plain, plain.desc.off_work, plain.desc.num_work)


def test_prefix_pass_of_unequal_groups_is_cut_into_pieces_of_one_length():
    # The decode groups' prefixes run 8192..32768 keys (64..256 K tiles per item).  The
    # planner may cut every item into the same number of pieces, or every item into
    # pieces of about one length; whichever it takes, each item's pieces cover its K
    # tiles once, in order, each piece writes its own partial slot, and the pieces are
    # the fewest that keep the simulated schedule within 2 % of the best.  Here the
    # equal-length cut wins: all pieces within 1.5x of each other (equal counts per item
    # would leave 2x between the longest and the shortest).
    wl = synth.make_workload(6, values=False)
    b = wl.batches[0]
    tab = sa.SegTable.build(None, b.seg_starts, b.seg_lens, wl.num_slots, True,
                            sa.MODE_DECODE | sa.SHARE_PREFIX, wl.q_heads, wl.kv_heads,
                            wl.head_dim)
    d = tab.desc
    w = arr(tab, d.off_group_work, d.num_group_work, 16)
    lens = w[:, 4] - w[:, 3]
    assert (lens >= 8).all()
    items = {}
    for row in w:
        items.setdefault((row[0], row[1], row[2]), []).append(row)
    totals = []
    for rows in items.values():
        rows = sorted(rows, key=lambda r: r[3])
        assert rows[0][3] == 0
        assert all(a[4] == b_[3] for a, b_ in zip(rows, rows[1:]))
        totals.append(rows[-1][4])
    assert max(totals) >= 2 * min(totals) - 1  # the items really differ in length
    assert lens.max() <= 1.5 * lens.min()
    assert sorted(w[:, 5].tolist()) == list(range(d.num_group_parts))
