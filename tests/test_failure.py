"""Failure detection without a GPU fault: a wait that nothing completes must give up
after its limit, surface as the device error word, and leave the context usable --
for a lone diagnostic warp, and for the prefill kernel itself when its producer
withholds a K tile (the stall test switch), which exercises the kernel's drain of
the copies and MMAs already in flight and its release of tensor memory."""
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa

from helpers import compare, random_case, run_cuda, shared_case, shared_values

S = sa.STATUS


def test_wait_selftest_rejects_out_of_range_limits():
    # host-side check only; nothing is launched (no GPU needed)
    lib = sa.load_library()
    for bad in (0, -5, 1000001):
        assert lib.seg_attn_wait_selftest(bad, None) == S["INVALID_ARG"]
        assert lib.seg_attn_stall_test(-1, bad) == S["INVALID_ARG"]
    assert lib.seg_attn_stall_test(-1, 1000000) == 0  # the defaults
    for bad in (-1, 1000001):
        assert lib.seg_attn_order_test(bad) == S["INVALID_ARG"]
    assert lib.seg_attn_order_test(0) == 0  # off, the default


def _stall_case(q_per_req, hq=8, hkv=2, d=128):
    """Request 0 has 200 keys (2 K tiles), request 1 has 1000 (8 K tiles); non-causal, so
    every item of request 1 reaches K tile 2 and every item of request 0 stops short."""
    case = random_case(62, batch=2, hq=hq, hkv=hkv, d=d, causal=False, max_k=4)
    g = torch.Generator().manual_seed(63)
    S_ = 1700
    k = torch.full((S_, hkv, d), float("nan"))
    v = torch.full((S_, hkv, d), float("nan"))
    starts = [[10, 230], [600, 1300]]  # two segments per request, free (NaN) slots between
    lens = [[120, 80], [650, 350]]
    for ss, ll in zip(starts, lens):
        for s0, l in zip(ss, ll):
            k[s0:s0 + l] = torch.randn(l, hkv, d, generator=g)
            v[s0:s0 + l] = torch.randn(l, hkv, d, generator=g)
    case.update(q_lens=[q_per_req, q_per_req], seg_starts=starts, seg_lens=lens, num_slots=S_,
                k_pool=k.to(torch.bfloat16), v_pool=v.to(torch.bfloat16),
                q=torch.randn(2 * q_per_req, hq, d, generator=g).to(torch.bfloat16))
    return case


@pytest.mark.gpu
@pytest.mark.parametrize("variant", ["two-tile", "one-tile", "e4m3"])
def test_prefill_gives_up_on_a_withheld_tile_and_recovers(variant):
    """The producer stops before K tile 2: CTAs of request 1 (8 tiles) wait, give up after
    1 ms, drain and exit without writing their rows; CTAs of request 0 (2 tiles) finish.
    Afterwards the same process computes a normal prefill correctly."""
    from segmented_kv_cache_b200 import synth
    q_per_req = 20 if variant == "one-tile" else 50  # qpt = 128 / 4 = 32 queries per tile
    case = _stall_case(q_per_req)
    c = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    tab = sa.SegTable.build(case["q_lens"], case["seg_starts"], case["seg_lens"],
                            case["num_slots"], False, sa.MODE_PREFILL, 8, 2, 128).to("cuda")
    assert (tab.desc.num_single == tab.desc.num_work) == (variant == "one-tile")
    assert tab.workspace_bytes == 0  # no split pieces: each item is one CTA
    out = torch.full_like(c["q"], float("nan"))
    lse = torch.full(c["q"].shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    if variant == "e4m3":
        k8, v8, ks, vs = synth.fp8_pools(case["k_pool"], case["v_pool"])
        k8, v8, ks, vs = k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda()
        call = lambda: sa.seg_attn_prefill_fp8(c["q"], k8, v8, ks, vs, out, lse, tab.device,
                                               tab.desc, case["scale"], None)
        ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                            case["q"], k8.cpu(), v8.cpu(), ks.cpu(), vs.cpu(),
                                            case["scale"], False)
    else:
        call = lambda: sa.seg_attn_prefill(c["q"], c["k_pool"], c["v_pool"], out, lse, tab.device,
                                           tab.desc, case["scale"], None)
        ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                        case["q"], case["k_pool"], case["v_pool"], case["scale"],
                                        False)
    assert sa.seg_attn_take_device_error() == 0
    try:
        sa.seg_attn_stall_test(2, 1000)
        call()
        torch.cuda.synchronize()
    finally:
        sa.seg_attn_stall_test(-1, 1000000)
    assert sa.seg_attn_take_device_error() == 1
    assert sa.seg_attn_take_device_error() == 0
    n0 = q_per_req
    # request 0 finished normally; request 1's CTAs gave up and wrote nothing
    compare(out[:n0], lse[:n0], ref_o[:n0], ref_l[:n0], f"stall test {variant}: finished CTAs")
    assert torch.isnan(out[n0:].float()).all() and torch.isnan(lse[n0:]).all()
    # the context is intact: the same call without the stall matches the oracle everywhere
    out.fill_(float("nan"))
    lse.fill_(float("nan"))
    call()
    torch.cuda.synchronize()
    compare(out, lse, ref_o, ref_l, f"after the stall test ({variant})")
    assert sa.seg_attn_take_device_error() == 0


@pytest.mark.gpu
def test_stalled_wait_is_reported_and_the_context_survives():
    assert sa.seg_attn_take_device_error() == 0
    sa.seg_attn_wait_selftest(2000)  # 2 ms on a barrier nobody arrives on
    torch.cuda.synchronize()
    assert sa.seg_attn_take_device_error() == 1
    assert sa.seg_attn_take_device_error() == 0  # reading clears the word
    # the same process keeps computing correctly afterwards
    case = random_case(61, batch=2, hq=8, hkv=2, d=128, causal=True, max_k=700)
    c = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    out, lse, _ = run_cuda(c["q"], c["k_pool"], c["v_pool"], case["q_lens"], case["seg_starts"],
                           case["seg_lens"], case["num_slots"], True, sa.MODE_PREFILL,
                           case["scale"])
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                    case["q"], case["k_pool"], case["v_pool"], case["scale"], True)
    compare(out, lse, ref_o, ref_l, "after a reported stall")
    assert sa.seg_attn_take_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("variant", ["one-tile", "one-tile e4m3", "shared-prefix decode"])
def test_late_softmax_at_the_end_of_an_item_keeps_results(variant):
    """Every softmax warp of a one-tile item sleeps 30 us after signalling P of the item's
    last K tile (the order test switch), so the last P.V product has completed before the
    warp waits for it.  No wait may give up and the results must match the oracle: the
    end wait used to take that state for an earlier one and wait out its limit.  (The
    two-tile kernel waits for PV(i - 1) before it writes P(i), so it never meets it.)"""
    from segmented_kv_cache_b200 import synth
    if variant == "shared-prefix decode":
        # the pass over the shared prefixes runs the one-tile kernel on pieces of many K tiles
        reqs, q_lens, S_ = shared_case(3, B=8, decode=True, max_prefix=5000)
        case = shared_values(reqs, q_lens, S_, 64, 8, 128, seed=20)
        mode, causal = sa.MODE_DECODE | sa.SHARE_PREFIX, True
        q_arg = None
    else:
        case = _stall_case(20)  # qpt = 32: one query tile per item
        mode, causal = sa.MODE_PREFILL, False
        q_arg = case["q_lens"]
    c = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    assert sa.seg_attn_take_device_error() == 0
    try:
        sa.seg_attn_order_test(30000)
        if variant == "one-tile e4m3":
            tab = sa.SegTable.build(q_arg, case["seg_starts"], case["seg_lens"], case["num_slots"],
                                    causal, mode, 8, 2, 128).to("cuda")
            k8, v8, ks, vs = synth.fp8_pools(case["k_pool"], case["v_pool"])
            out = torch.full_like(c["q"], float("nan"))
            lse = torch.full(c["q"].shape[:2], float("nan"), dtype=torch.float32, device="cuda")
            sa.seg_attn_prefill_fp8(c["q"], k8.cuda(), v8.cuda(), ks.cuda(), vs.cuda(), out, lse,
                                    tab.device, tab.desc, case["scale"], None)
            ref_o, ref_l = oracle.attention_fp8(case["q_lens"], case["seg_starts"],
                                                case["seg_lens"], case["q"], k8, v8, ks, vs,
                                                case["scale"], causal)
        else:
            out, lse, tab = run_cuda(c["q"], c["k_pool"], c["v_pool"], q_arg, case["seg_starts"],
                                     case["seg_lens"], case["num_slots"], causal, mode,
                                     case["scale"])
            ref_o, ref_l = oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"],
                                            case["q"], case["k_pool"], case["v_pool"],
                                            case["scale"], causal)
        torch.cuda.synchronize()
    finally:
        sa.seg_attn_order_test(0)
    if variant.startswith("one-tile"):
        assert tab.desc.num_single == tab.desc.num_work
    if variant == "shared-prefix decode":
        assert tab.desc.shared == 1
    assert sa.seg_attn_take_device_error() == 0
    compare(out, lse, ref_o, ref_l, f"late softmax ({variant})")
