"""Segment allocator (host C++) against the list-based model of its policy: exact slots,
exact segment lists and statistics after every operation of random workloads."""
import random

import numpy as np
import pytest

import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import _build

from pool_model import PoolModel


@pytest.fixture(scope="module", autouse=True)
def built():
    _build.build()


@pytest.mark.parametrize("seed", range(8))
def test_random_workload_matches_model(seed):
    rng = random.Random(seed)
    n = rng.choice([64, 300, 1000])
    pool, model = sa.SegPool(n), PoolModel(n)
    live = []
    for step in range(400):
        op = rng.random()
        if op < 0.6 or not live:
            seq = rng.choice(live) if live and rng.random() < 0.7 else rng.randrange(10**6)
            k = rng.choice([0, 1, 1, 2, 3, rng.randrange(1, n // 4 + 2)])
            want = model.append(seq, k)
            if want is None:
                with pytest.raises(sa.SegAttnError) as e:
                    pool.append(seq, k)
                assert e.value.code == sa.STATUS["NO_SPACE"]
                continue
            got = pool.append(seq, k).tolist()
            assert got == want, (step, seq, k)
            if seq not in live:
                live.append(seq)
        else:
            seq = live.pop(rng.randrange(len(live)))
            pool.release(seq)
            model.release(seq)
        assert pool.stats() == model.stats(), step
        for s in live:
            st, ln = pool.segments(s)
            assert list(zip(st, ln)) == model.seqs[s]
    # release everything: one free run of the whole pool
    for s in live:
        pool.release(s)
    assert pool.stats() == dict(num_slots=n, free_slots=n, free_runs=1, largest_free_run=n,
                                sequences=0, segments=0)


def test_in_place_growth_keeps_one_segment():
    pool = sa.SegPool(100)
    a = pool.append(1, 10)
    b = pool.append(1, 5)
    assert a.tolist() == list(range(10)) and b.tolist() == list(range(10, 15))
    assert pool.segments(1) == ([0], [15])
    pool.append(2, 3)  # occupies 15..17, so seq 1 cannot grow in place any more
    c = pool.append(1, 4)
    st, ln = pool.segments(1)
    assert len(st) == 2 and st[0] == 0 and ln == [15, 4] and c.tolist() == list(range(st[1], st[1] + 4))


def test_best_fit_and_coalescing():
    pool = sa.SegPool(100)
    for s, k in [(1, 10), (2, 5), (3, 20), (4, 3), (5, 62)]:
        pool.append(s, k)
    pool.release(2)   # free 10..14  (5 slots)
    pool.release(4)   # free 35..37  (3 slots)
    assert pool.append(6, 3).tolist() == [35, 36, 37]   # smallest run that fits
    pool.release(6)
    pool.release(3)   # 15..34 freed and merged with 10..14 and 35..37 -> 10..37
    assert pool.stats()["free_runs"] == 1 and pool.stats()["largest_free_run"] == 28


def test_no_space_leaves_pool_unchanged():
    pool = sa.SegPool(10)
    pool.append(1, 8)
    before = pool.stats()
    with pytest.raises(sa.SegAttnError) as e:
        pool.append(2, 3)
    assert e.value.code == sa.STATUS["NO_SPACE"]
    assert pool.stats() == before


def test_bad_arguments():
    pool = sa.SegPool(10)
    with pytest.raises(sa.SegAttnError):
        pool.release(12345)
    with pytest.raises(sa.SegAttnError):
        pool.append(1, -1)
    with pytest.raises(sa.SegAttnError):
        sa.SegPool(-1)
