"""Failure detection without a GPU fault: a wait that nothing completes must give up
after its limit, surface as the device error word, and leave the context usable."""
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa

from helpers import compare, random_case, run_cuda

S = sa.STATUS


def test_wait_selftest_rejects_out_of_range_limits():
    # host-side check only; nothing is launched (no GPU needed)
    lib = sa.load_library()
    for bad in (0, -5, 1000001):
        assert lib.seg_attn_wait_selftest(bad, None) == S["INVALID_ARG"]


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
