"""The C ABI without a GPU: the library loads, exports what include/*.h declares,
and the host-side table builder / argument checks behave as documented."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest
import torch

import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
S = sa.STATUS


@pytest.fixture(scope="module", autouse=True)
def built_library():
    _build.build()
    return sa.load_library()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(seg_(?:attn|la)_\w+)\s*\(",
                            text, re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(built_library):
    names = declared_functions()
    assert {"seg_attn_build_table", "seg_attn_prefill", "seg_attn_decode",
            "seg_attn_workspace_size", "seg_attn_status_string", "seg_la_build_table",
            "seg_la_prefill", "seg_la_decode", "seg_la_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(built_library, n), n


def test_status_strings_and_version():
    for name, code in S.items():
        assert sa.seg_attn_status_string(code)
    assert sa.seg_attn_status_string(12345) == "unknown status"
    assert sa.seg_attn_version() >= 100


def build(q_lens, segs, num_slots=100, causal=True, mode=sa.MODE_PREFILL, hq=8, hkv=2, d=128):
    starts = [[s for s, _ in r] for r in segs]
    lens = [[l for _, l in r] for r in segs]
    return sa.SegTable.build(q_lens, starts, lens, num_slots, causal, mode, hq, hkv, d)


def code_of(fn):
    with pytest.raises(sa.SegAttnError) as e:
        fn()
    return e.value.code


def test_validation_errors():
    assert code_of(lambda: build([2], [[(95, 10)]])) == S["SEGMENT_OOB"]
    assert code_of(lambda: build([2], [[(-1, 3)]])) == S["SEGMENT_OOB"]
    assert code_of(lambda: build([2], [[(10, 5), (12, 4)]])) == S["SEGMENT_OVERLAP"]
    assert code_of(lambda: build([5], [[(10, 4)]])) == S["QLEN_GT_KLEN"]
    # non-causal prefill may have more queries than keys
    build([5], [[(10, 4)]], causal=False)
    assert code_of(lambda: build([2], [[(10, -1)]])) == S["INVALID_ARG"]
    assert code_of(lambda: build([-1], [[(10, 4)]])) == S["INVALID_ARG"]
    assert code_of(lambda: build([1], [[(10, 4)]], hq=6, hkv=4)) == S["INVALID_ARG"]
    assert code_of(lambda: build([1], [[(10, 4)]], d=96)) == S["UNSUPPORTED"]
    assert code_of(lambda: build([1], [[(10, 4)]], hq=6, hkv=2)) == S["UNSUPPORTED"]  # G=3
    # decode covers groups above 8 with sibling CTAs of 8 heads each; 256 is past the limit
    build([1], [[(10, 4)]], hq=32, hkv=2, mode=sa.MODE_DECODE)
    build([1], [[(10, 4)]], hq=128, hkv=1, mode=sa.MODE_DECODE)
    assert code_of(lambda: build([1], [[(10, 4)]], hq=256, hkv=1, mode=sa.MODE_DECODE)) == S["UNSUPPORTED"]
    assert code_of(lambda: build([1], [[(10, 4)]], hq=256, hkv=1)) == S["UNSUPPORTED"]
    assert code_of(lambda: build([2], [[(10, 4)]], mode=sa.MODE_DECODE)) == S["INVALID_ARG"]
    # the same slots in two requests are legal (shared read-only prefix)
    build([1, 1], [[(10, 4)], [(10, 4)]])
    # int32 pool row index limit
    assert code_of(lambda: build([1], [[(0, 4)]], num_slots=2**30, hkv=2)) == S["UNSUPPORTED"]


def test_size_query_and_small_buffer():
    lib = sa.load_library()
    desc = sa.seg_attn_table_desc()
    q = np.array([3], np.int32)
    c = np.array([1], np.int32)
    st = np.array([4], np.int32)
    ln = np.array([7], np.int32)
    P = lambda a: ctypes.c_void_p(a.ctypes.data)
    rc = lib.seg_attn_build_table(1, P(q), P(c), P(st), P(ln), 20, 1, 0, 8, 2, 128, None, 0,
                                  ctypes.byref(desc))
    assert rc == 0 and desc.table_bytes > 0 and desc.magic == 0x53454741
    buf = np.zeros(desc.table_bytes // 4 - 1, np.int32)
    rc = lib.seg_attn_build_table(1, P(q), P(c), P(st), P(ln), 20, 1, 0, 8, 2, 128, P(buf),
                                  buf.nbytes, ctypes.byref(desc))
    assert rc == S["BUFFER_TOO_SMALL"]
    assert lib.seg_attn_build_table(1, P(q), P(c), P(st), P(ln), 20, 1, 0, 8, 2, 128, None, 0,
                                    None) == S["INVALID_ARG"]


def view(tab, off, n):
    return tab.host[off: off + n].tolist()


def test_prefill_table_contents():
    tab = build([3, 0, 40], [[(50, 2), (10, 5)], [(0, 3)], [(20, 20), (60, 30)]], num_slots=100,
                hq=8, hkv=2)
    d = tab.desc
    assert d.batch == 3 and d.total_q == 43 and d.total_k == 60 and d.num_segments == 5
    assert view(tab, d.off_q_offsets, 4) == [0, 3, 3, 43]
    assert view(tab, d.off_k_lens, 3) == [7, 3, 50]
    assert view(tab, d.off_seg_offsets, 4) == [0, 2, 3, 5]
    assert view(tab, d.off_seg_start, 5) == [50, 10, 0, 20, 60]
    assert view(tab, d.off_seg_kstart, 5) == [0, 2, 0, 0, 20]
    assert view(tab, d.off_seg_len, 5) == [2, 5, 3, 20, 30]
    assert d.off_work % 4 == 0 and d.queries_per_tile == 32  # 128 rows / group 4
    work = np.array(view(tab, d.off_work, 16 * d.num_work)).reshape(-1, 16)
    # request 0: one pair x 2 kv heads; request 2: 40 queries -> 1 pair (64 per pair) x 2 heads
    assert len(work) == 4 and sorted(set(work[:, 0])) == [0, 2]
    # causal tile count: last query of request 2 sees all 50 keys -> tiles [0, 1), unsplit
    assert all(w[3] == 0 and w[4] == 1 and w[5] == -1 for w in work)
    # request words of each row: end of its segments, first query row, queries, keys,
    # segment of the first key
    q_off, k_len, s_off = [0, 3, 3, 43], [7, 3, 50], [0, 2, 3, 5]
    for w in work:
        r = w[0]
        assert list(w[7:12]) == [s_off[r + 1], q_off[r], q_off[r + 1] - q_off[r], k_len[r], s_off[r]]
        # first K tile in one segment: its first slot; otherwise -1 (here every request's
        # first tile spans more than one segment, or the request has no tile at all)
        assert w[12] == -1 and list(w[13:16]) == [0, 0, 0]


def test_prefill_first_segment_of_split_pieces():
    # 4000 keys over segments with zero-length ones in between; the single item is cut
    # into pieces along its 32 K tiles, each row names the segment of its first key as
    # the device walk finds it: the last segment whose logical start is <= that key
    lens = [0, 300, 0, 1200, 0, 0, 2500]
    starts = [0, 10, 400, 500, 2000, 2000, 3000]
    tab = build([1], [list(zip(starts, lens))], num_slots=6000, causal=False, hq=8, hkv=1)
    d = tab.desc
    work = np.array(view(tab, d.off_work, 16 * d.num_work)).reshape(-1, 16)
    assert d.num_work > 1 and d.num_merge == 1  # split into several pieces
    kstart = np.cumsum([0] + lens)[:-1]
    for w in work:
        j = w[3] * 128
        want = max(i for i in range(len(lens)) if kstart[i] <= j)
        assert w[11] == want and w[7] == len(lens) and list(w[8:11]) == [0, 1, 4000]
        # the slot of the first key when the piece's first tile lies inside that segment
        inside = j + 128 <= kstart[want] + lens[want]
        assert w[12] == (starts[want] + j - kstart[want] if inside else -1)


def test_decode_chunks_cover_each_request():
    k = [5000, 1, 0, 2049]
    segs = [[(0, 5000)], [(6000, 1)], [], [(7000, 1000), (9000, 1049)]]
    tab = build([1] * 4, segs, num_slots=20000, mode=sa.MODE_DECODE, hq=8, hkv=1)
    d = tab.desc
    L = d.chunk_len
    assert L >= 256 and d.workspace_bytes > 0
    work = np.array(view(tab, d.off_work, 4 * d.num_work)).reshape(-1, 4)
    rc = view(tab, d.off_req_chunks, 5)
    for r in range(4):
        w = work[rc[r]: rc[r + 1]]
        assert (w[:, 0] == r).all()
        assert w[0, 1] == 0 and w[-1, 2] == k[r]
        assert (w[1:, 1] == w[:-1, 2]).all()
        assert (w[:, 3] == len(w)).all()
        assert ((w[:, 2] - w[:, 1]) <= L).all()


def test_compute_calls_reject_bad_arguments_before_any_launch():
    # all of these fail host-side checks; no CUDA call is made
    tab = build([2], [[(10, 5)]])
    fake = torch.zeros(16, dtype=torch.uint8)
    p = lambda: ctypes.c_void_p(fake.data_ptr())
    lib = sa.load_library()
    desc = tab.desc
    call = lambda fn, scale, dsc=desc, q=None, ws=None, wsb=0: getattr(lib, fn)(
        q if q is not None else p(), p(), p(), p(), None, p(), ctypes.byref(dsc), scale,
        ws, wsb, None)
    assert call("seg_attn_prefill", 0.0) == S["INVALID_ARG"]
    assert call("seg_attn_prefill", float("nan")) == S["INVALID_ARG"]
    assert call("seg_attn_decode", 0.1) == S["INVALID_ARG"]  # table built for prefill
    assert call("seg_attn_prefill", 0.1, q=ctypes.c_void_p(fake.data_ptr() + 2)) == S["INVALID_ARG"]
    bad = sa.seg_attn_table_desc.from_buffer_copy(desc)
    bad.magic = 0
    assert call("seg_attn_prefill", 0.1, dsc=bad) == S["INVALID_ARG"]
    dtab = build([1, 1], [[(0, 3000)], [(4000, 10)]], num_slots=5000, mode=sa.MODE_DECODE, hq=8,
                 hkv=1)
    assert dtab.desc.workspace_bytes > 0
    assert call("seg_attn_decode", 0.1, dsc=dtab.desc) == S["WORKSPACE"]
    assert call("seg_attn_decode", 0.1, dsc=dtab.desc, ws=p(), wsb=16) == S["WORKSPACE"]


def test_empty_batch_is_a_noop():
    tab = build([], [], num_slots=0)
    assert tab.desc.num_work == 0 and tab.desc.total_q == 0
    lib = sa.load_library()
    rc = lib.seg_attn_prefill(None, None, None, None, None, None, ctypes.byref(tab.desc), 0.1,
                              None, 0, None)
    assert rc == 0


def test_prefill_split_plan_covers_every_item_once():
    # one long request, few query tiles: the planner cuts items along their keys
    tab = build([64], [[(0, 20000)]], num_slots=20000, hq=16, hkv=2)
    d = tab.desc
    assert d.num_merge > 0 and d.num_parts > d.num_merge and d.workspace_bytes > 0
    work = np.array(view(tab, d.off_work, 16 * d.num_work)).reshape(-1, 16)
    merge = np.array(view(tab, d.off_merge, 8 * d.num_merge)).reshape(-1, 8)
    seen_slots = set()
    for r, g, q0, slot0, parts, *_ in merge:
        visible = min(20000, 20000 - 64 + min(64, q0 + 32))  # 16 queries per tile, 2 tiles
        tiles = (visible + 127) // 128
        pieces = work[(work[:, 0] == r) & (work[:, 1] == g) & (work[:, 2] == q0)]
        assert len(pieces) == parts
        pieces = pieces[np.argsort(pieces[:, 3])]
        assert pieces[0, 3] == 0 and pieces[-1, 4] == tiles
        assert (pieces[1:, 3] == pieces[:-1, 4]).all()
        assert sorted(pieces[:, 5]) == list(range(slot0, slot0 + parts))
        seen_slots |= set(pieces[:, 5].tolist())
    assert seen_slots == set(range(d.num_parts))
    # longest pieces first
    lens = work[:, 4] - work[:, 3]
    assert list(lens) == sorted(lens, reverse=True)
    rows = 256
    assert d.workspace_bytes >= d.num_parts * rows * (d.head_dim + 1) * 4


def test_prefill_without_split_needs_no_workspace():
    tab = build([40, 3], [[(20, 20), (60, 30)], [(0, 7)]], num_slots=100, hq=8, hkv=2)
    d = tab.desc
    assert d.num_merge == 0 and d.num_parts == 0 and d.workspace_bytes == 0
    work = np.array(view(tab, d.off_work, 16 * d.num_work)).reshape(-1, 16)
    assert (work[:, 5] == -1).all() and (work[:, 3] == 0).all()


def test_prefill_one_tile_kernel_only_for_all_single_tile_passes():
    # G = 8: 16 queries per 128-row tile, 32 per item.
    # Requests of 10 and 7 queries: every item holds queries in its first tile only.
    tab = build([10, 7], [[(0, 300)], [(400, 200)]], num_slots=900, hq=16, hkv=2)
    d = tab.desc
    work = np.array(view(tab, d.off_work, 16 * d.num_work)).reshape(-1, 16)
    assert d.num_single == d.num_work == 4 and (work[:, 6] == 1).all()
    lens = work[:, 4] - work[:, 3]
    assert list(lens) == sorted(lens, reverse=True)
    # a request of 40 queries adds an item with two query tiles: one two-tile launch
    tab = build([40, 10, 7], [[(0, 300)], [(400, 200)], [(700, 100)]], num_slots=900, hq=16,
                hkv=2)
    d = tab.desc
    work = np.array(view(tab, d.off_work, 16 * d.num_work)).reshape(-1, 16)
    assert d.num_single == 0 and (work[:, 6] == 0).all()


def test_fp8_calls_reject_missing_or_misaligned_scales():
    # host-side checks of the FP8 entry points; nothing is launched
    fake = torch.zeros(16, dtype=torch.uint8)
    p = lambda: ctypes.c_void_p(fake.data_ptr())
    lib = sa.load_library()
    for fn, mode in (("seg_attn_prefill_fp8", sa.MODE_PREFILL),
                     ("seg_attn_decode_fp8", sa.MODE_DECODE)):
        tab = build([1] if mode == sa.MODE_DECODE else [2], [[(10, 5)]], mode=mode)
        call = lambda ks, vs, dsc: getattr(lib, fn)(p(), p(), p(), ks, vs, p(), None, p(),
                                                    ctypes.byref(dsc), 0.1, p(), 1 << 20, None)
        assert call(None, p(), tab.desc) == S["INVALID_ARG"]
        assert call(p(), None, tab.desc) == S["INVALID_ARG"]
        assert call(ctypes.c_void_p(fake.data_ptr() + 2), p(), tab.desc) == S["INVALID_ARG"]
