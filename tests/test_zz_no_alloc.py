"""seg_attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers (a plugin inside a runtime that owns all device memory, a serving
loop that must not call cudaMalloc once running) cannot provide the split-K
workspace.  The no-allocation entry point keeps that scratch in a fixed array
inside the library.  These checks call it through the C ABI twice in a row and
compare each result with seg_attn_decode given a caller-allocated workspace, and
with the fp64 oracle; plain and shared-prefix decode tables (whose scratch holds
the prefix pass's partials as well) are both covered.

The file name sorts last so a run that stops at the first failure has already
run every other test.
"""
import ctypes

import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa

from helpers import (LSE_REL, MAX_ABS, MEAN_ABS, compare, random_case, run_cuda, shared_case,
                     shared_values)

pytestmark = pytest.mark.gpu

NOALLOC_LIMIT = 64 << 20


def _noalloc_fn():
    fn = sa.load_library().seg_attn_decode_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [P, P, P, P, P, P, ctypes.POINTER(sa.seg_attn_table_desc), ctypes.c_float, P]
    fn.restype = ctypes.c_int
    return fn


def _decode_noalloc(case, mode=sa.MODE_DECODE):
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    tab = sa.SegTable.build(None, case["seg_starts"], case["seg_lens"], case["num_slots"], True,
                            mode, dev["q"].shape[1], dev["k_pool"].shape[1],
                            dev["q"].shape[2]).to("cuda")
    out = torch.full_like(dev["q"], float("nan"))
    lse = torch.full(dev["q"].shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = _noalloc_fn()(P(dev["q"]), P(dev["k_pool"]), P(dev["v_pool"]), P(out), P(lse),
                       P(tab.device), ctypes.byref(tab.desc), case["scale"],
                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, sa.seg_attn_status_string(rc)
    return out, lse, tab


def _reference(case, mode=sa.MODE_DECODE):
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    out, lse, _ = run_cuda(dev["q"], dev["k_pool"], dev["v_pool"], None, case["seg_starts"],
                           case["seg_lens"], case["num_slots"], True, mode, case["scale"])
    return out, lse


def _close(out, lse, ref_out, ref_lse):
    err = (out.double() - ref_out.double()).abs()
    assert torch.isfinite(out.float()).all()
    assert float(err.max()) <= MAX_ABS and float(err.mean()) <= MEAN_ABS
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(lse), fin)
    rel = (lse[fin].double() - ref_lse[fin].double()).abs() / ref_lse[fin].double().abs().clamp(min=1)
    assert rel.numel() == 0 or float(rel.max()) <= LSE_REL


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    # two different batches, both long enough to be split into several chunks,
    # so the second call runs over the scratch the first one left behind
    first = random_case(501, batch=6, hq=64, hkv=8, d=128, causal=True, max_k=9000, nseg_max=6,
                        q_mode="decode")
    second = random_case(502, batch=3, hq=16, hkv=2, d=64, causal=True, max_k=5000, nseg_max=3,
                         q_mode="decode")
    results = []
    for case in (first, second):
        out, lse, tab = _decode_noalloc(case)
        assert 0 < tab.workspace_bytes <= NOALLOC_LIMIT
        results.append((out, lse))
    torch.cuda.synchronize()
    for case, (out, lse) in zip((first, second), results):
        ref_out, ref_lse = _reference(case)
        torch.cuda.synchronize()
        _close(out, lse, ref_out, ref_lse)
    # and the first call straight against the fp64 oracle
    o, l = oracle.attention(first["q_lens"], first["seg_starts"], first["seg_lens"], first["q"],
                            first["k_pool"], first["v_pool"], first["scale"], True)
    compare(results[0][0], results[0][1], o, l, "no-allocation decode vs oracle")
    assert sa.seg_attn_take_device_error() == 0


def test_noalloc_shared_prefix_tables_on_two_calls_in_a_row():
    # A shared-prefix decode table lays out more scratch (the requests' own-key
    # partials, then the pass over the prefixes): two such tables in a row, each
    # checked against seg_attn_decode with a caller workspace and against the oracle.
    cases = []
    for seed, (hq, hkv, d) in ((3, (64, 8, 128)), (5, (16, 2, 64))):
        reqs, q, S = shared_case(seed, B=8, decode=True, max_prefix=5000)
        cases.append(shared_values(reqs, q, S, hq, hkv, d, seed=seed + 17))
    mode = sa.MODE_DECODE | sa.SHARE_PREFIX
    results = []
    for case in cases:
        out, lse, tab = _decode_noalloc(case, mode)
        assert tab.desc.shared == 1 and 0 < tab.workspace_bytes <= NOALLOC_LIMIT
        results.append((out, lse))
    torch.cuda.synchronize()
    for case, (out, lse) in zip(cases, results):
        ref_out, ref_lse = _reference(case, mode)
        torch.cuda.synchronize()
        _close(out, lse, ref_out, ref_lse)
        o, l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"], case["q"],
                                case["k_pool"], case["v_pool"], case["scale"], True)
        compare(out, lse, o, l, "no-allocation shared-prefix decode vs oracle")
    assert sa.seg_attn_take_device_error() == 0


def test_noalloc_rejects_tables_needing_more_scratch_than_the_array():
    # 2048 requests of 8192 keys with 64 query heads need more than 64 MiB of partials
    n = 2048
    tab = sa.SegTable.build(None, [[0]] * n, [[8192]] * n, 8192, True, sa.MODE_DECODE, 64, 8, 128)
    assert tab.workspace_bytes > NOALLOC_LIMIT
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    P = ctypes.c_void_p(dummy.data_ptr())
    rc = _noalloc_fn()(P, P, P, P, None, P, ctypes.byref(tab.desc), 0.1, None)
    assert rc == sa.STATUS["WORKSPACE"]
