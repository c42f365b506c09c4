"""Segment linear attention boundary without a GPU: table builder (chunk list, slot
checks) and argument checks of the compute calls."""
import ctypes

import numpy as np
import pytest

import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import _build

S = sa.STATUS
H, D = 4, 128


@pytest.fixture(scope="module", autouse=True)
def built_library():
    _build.build()
    return sa.load_library()


def arr(tab, off, n, width=1):
    a = tab.host[off: off + n * width].numpy().copy()
    return a.reshape(-1, width) if width > 1 else a


def code_of(fn):
    with pytest.raises(sa.SegAttnError) as e:
        fn()
    return e.value.code


def test_prefill_chunk_list():
    q_lens = [0, 1, 128, 129, 300]
    tab = sa.LATable.build(q_lens, [-1, 0, -1, 2, 3], [5, 0, 1, 2, 4], 6, sa.MODE_PREFILL, H, D)
    d = tab.desc
    assert d.chunk_len == 128 and d.num_chunks == 0 + 1 + 1 + 2 + 3 and d.total_q == 558
    ch = arr(tab, d.off_chunks, d.num_chunks, 4)
    q_off = np.concatenate([[0], np.cumsum(q_lens)])
    want = []
    for r, n in enumerate(q_lens):
        for i, t0 in enumerate(range(0, n, 128)):
            want.append([r, q_off[r] + t0, min(128, n - t0), i])
    assert ch.tolist() == want
    assert arr(tab, d.off_req_chunks, 6).tolist() == [0, 0, 1, 2, 4, 7]
    assert arr(tab, d.off_q_offsets, 6).tolist() == q_off.tolist()
    units = d.num_chunks * H
    assert d.workspace_bytes >= units * (D * D * 4 + D * D * 2 + 4)


def test_decode_table_needs_no_workspace():
    tab = sa.LATable.build(None, [0, 1, -1], [0, 1, 2], 3, sa.MODE_DECODE, H, D)
    assert tab.desc.workspace_bytes == 0 and tab.desc.total_q == 3
    assert code_of(lambda: sa.LATable.build([2], [0], [0], 1, sa.MODE_DECODE, H, D)) == \
        S["INVALID_ARG"]


def test_slot_checks():
    build = lambda i, o, n=4: sa.LATable.build([3] * len(i), i, o, n, sa.MODE_PREFILL, H, D)
    assert code_of(lambda: build([4], [0])) == S["SEGMENT_OOB"]
    assert code_of(lambda: build([0], [-2])) == S["SEGMENT_OOB"]
    assert code_of(lambda: build([0, 1], [2, 2])) == S["SEGMENT_OVERLAP"]   # one slot, two writers
    assert code_of(lambda: build([0, 1], [1, 3])) == S["SEGMENT_OVERLAP"]   # read of a written slot
    build([0, 1], [0, 1])        # each request updates its own slot in place
    build([0, 0], [2, 3])        # two requests fork from one state
    build([-1, -1], [-1, 3])     # a dropped final state
    assert code_of(lambda: sa.LATable.build([3], [0], [0], 1, sa.MODE_PREFILL, H, 64)) == \
        S["UNSUPPORTED"]


def test_compute_calls_check_arguments_before_launching():
    lib = sa.load_library()
    tab = sa.LATable.build([3], [-1], [0], 1, sa.MODE_PREFILL, H, D)
    p = ctypes.c_void_p(256)  # never dereferenced: the checks fail first
    dec = sa.LATable.build(None, [-1], [0], 1, sa.MODE_DECODE, H, D)
    # wrong mode
    rc = lib.seg_la_decode(p, p, p, p, p, p, p, ctypes.byref(tab.desc), 0.1, None)
    assert rc == S["INVALID_ARG"]
    rc = lib.seg_la_prefill(p, p, p, p, p, p, p, ctypes.byref(dec.desc), 0.1, p, 1 << 30, None)
    assert rc == S["INVALID_ARG"]
    # misaligned q, missing workspace
    rc = lib.seg_la_prefill(ctypes.c_void_p(258), p, p, p, p, p, p, ctypes.byref(tab.desc), 0.1,
                            p, 1 << 30, None)
    assert rc == S["INVALID_ARG"]
    rc = lib.seg_la_prefill(p, p, p, p, p, p, p, ctypes.byref(tab.desc), 0.1, None, 0, None)
    assert rc == S["WORKSPACE"]
    # empty batch is a no-op
    empty = sa.LATable.build([], [], [], 0, sa.MODE_PREFILL, H, D)
    assert lib.seg_la_prefill(None, None, None, None, None, None, None, ctypes.byref(empty.desc),
                              0.1, None, 0, None) == 0
