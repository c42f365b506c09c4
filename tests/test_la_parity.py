"""GPU parity of segment linear attention (simple GLA) against the fp64 oracle.

Tolerances, from the arithmetic.  Outputs are rounded to bf16, whose relative
rounding error is up to 2^-8 of the value; linear-attention outputs are not
bounded like a softmax average (a row can be several times the rms), so the
bound is per element, a relative part for that rounding plus an absolute part
scaled by the size of the reference:
  prefill:  |err| <= 2^-7 |ref| + 2e-2 rms(ref),  mean |err| <= 2e-3 rms(ref)
            (its products take bf16 operands -- the decay-weighted scores, the
            decay-scaled keys and the state entering a chunk, each rounded with
            relative error <= 2^-8 -- with fp32 accumulation: a per-element error
            of about 0.2 % of the rms, whose maximum over the ~2M outputs of a
            1024-token, 16-head call reaches ~5 sigma; 2e-2 rms is the 2e-2
            max-abs bound of the softmax path scaled to the size of the output;
            the same bound holds for the fp32 states it writes);
  decode:   output |err| <= 2^-8 |ref| + 1e-4 rms(ref) (fp32 arithmetic, then
            the bf16 rounding), state |err| <= 1e-5 rms(ref) (fp32 only)."""
import math

import numpy as np
import pytest
import torch

import oracle
import segmented_kv_cache_b200 as sa
from segmented_kv_cache_b200 import synth

pytestmark = pytest.mark.gpu

PREFILL = dict(rtol=2.0 ** -7, atol=2e-2, mean=2e-3)
DECODE_OUT = dict(rtol=2.0 ** -8, atol=1e-4, mean=2e-3)
DECODE_STATE = dict(rtol=0.0, atol=1e-5, mean=1e-6)


def check(got, ref, what, rtol=PREFILL["rtol"], atol=PREFILL["atol"], mean=PREFILL["mean"]):
    got = got.detach().double().cpu()
    assert torch.isfinite(got).all(), f"{what}: non-finite"
    if ref.numel() == 0:
        return 0.0
    rms = max(float(ref.pow(2).mean().sqrt()), 1e-30)
    err = (got - ref).abs()
    bound = rtol * ref.abs() + atol * rms
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: error {worst:.3f} x the bound (max err {float(err.max())}, rms {rms})"
    assert float(err.mean()) <= mean * rms, f"{what}: mean {float(err.mean())} vs rms {rms}"
    return worst


def run(w, mode=None, device="cuda"):
    """One call through the C ABI; returns (out, state pool after the call)."""
    mode = mode if mode is not None else (sa.MODE_PREFILL if w.mode == "prefill" else sa.MODE_DECODE)
    tab = sa.LATable.build(w.q_lens if mode == sa.MODE_PREFILL else None, w.in_slot, w.out_slot,
                           w.state_pool.shape[0], mode, w.heads, w.head_dim).to(device)
    q, k, v, g = (x.to(device) for x in (w.q, w.k, w.v, w.g))
    pool = w.state_pool.to(device).clone()
    out = torch.full_like(q, float("nan"))
    if mode == sa.MODE_PREFILL:
        ws = torch.empty(max(1, tab.workspace_bytes), dtype=torch.uint8, device=device)
        sa.seg_la_prefill(q, k, v, g, out, pool, tab.device, tab.desc, w.scale, ws)
    else:
        sa.seg_la_decode(q, k, v, g, out, pool, tab.device, tab.desc, w.scale)
    torch.cuda.synchronize()
    assert sa.seg_attn_take_device_error() == 0
    return out, pool


def reference(w):
    return oracle.linear_attention(w.q_lens, w.q.cpu(), w.k.cpu(), w.v.cpu(), w.g.cpu(), w.scale,
                                   w.state_pool.cpu(), w.in_slot)


def check_states(pool, w, ref_state, what, **tol):
    pool = pool.cpu()
    for r, o in enumerate(w.out_slot):
        if o >= 0:
            check(pool[o], ref_state[r], f"{what} state r{r}", **tol)
    # slots nobody writes are untouched
    written = {o for o in w.out_slot if o >= 0}
    for s in range(pool.shape[0]):
        if s not in written:
            assert torch.equal(pool[s], w.state_pool[s].cpu()), f"{what}: slot {s} changed"


@pytest.mark.parametrize("seed", [0, 1])
def test_prefill_varlen_with_states(seed):
    # ragged chunks, an empty request, one token, exact multiples of 128
    q_lens = [0, 1, 127, 128, 129, 300]
    w = synth.make_la_workload("custom", seed=seed, heads=4, q_lens=q_lens, fresh=False)
    w.in_slot = [w.in_slot[0], -1, w.in_slot[2], -1, w.in_slot[4], w.in_slot[5]]
    w.out_slot = list(w.out_slot[:5]) + [-1]  # the last request drops its final state
    out, pool = run(w, sa.MODE_PREFILL)
    ref_o, ref_s = reference(w)
    check(out, ref_o, f"prefill s{seed} out")
    check_states(pool, w, ref_s, f"prefill s{seed}")


def test_prefill_strong_and_no_decay():
    w = synth.make_la_workload("custom", seed=3, heads=2, q_lens=[200, 90], fresh=False)
    w.g[:200] = 0.0      # no decay over a long chunk: the state only grows
    w.g[200:] = -4.0     # exp(-4) per token: almost a reset
    out, pool = run(w, sa.MODE_PREFILL)
    ref_o, ref_s = reference(w)
    check(out[:200], ref_o[:200], "no decay out")
    check(out[200:], ref_o[200:], "strong decay out")
    check_states(pool, w, ref_s, "decay extremes")


def test_prefill_in_two_calls_through_the_pool():
    w = synth.make_la_workload("custom", seed=4, heads=4, q_lens=[300], fresh=False)
    one, pool_one = run(w, sa.MODE_PREFILL)
    a = synth.make_la_workload("custom", seed=4, heads=4, q_lens=[300], fresh=False)
    first = synth.LAWorkload(**{**a.__dict__, "q_lens": [150], "q": a.q[:150], "k": a.k[:150],
                                "v": a.v[:150], "g": a.g[:150]})
    o1, pool1 = run(first, sa.MODE_PREFILL)
    second = synth.LAWorkload(**{**a.__dict__, "q_lens": [150], "q": a.q[150:], "k": a.k[150:],
                                 "v": a.v[150:], "g": a.g[150:], "state_pool": pool1,
                                 "in_slot": a.out_slot})
    o2, pool2 = run(second, sa.MODE_PREFILL)
    ref_o, ref_s = reference(w)
    check(torch.cat([o1, o2]), ref_o, "split out")
    check(pool2[w.out_slot[0]], ref_s[0], "split state")
    check(one, ref_o, "one-call out")


def test_decode_random_states():
    w = synth.make_la_workload("custom", seed=5, heads=8, q_lens=[1] * 7, fresh=False)
    w.mode = "decode"
    w.in_slot[3] = -1   # a request with no state yet
    w.out_slot[5] = -1  # a request whose new state is dropped
    out, pool = run(w, sa.MODE_DECODE)
    ref_o, ref_s = reference(w)
    check(out, ref_o, "decode out", **DECODE_OUT)
    check_states(pool, w, ref_s, "decode", **DECODE_STATE)


@pytest.mark.parametrize("name", list(synth.LA_CONFIGS))
def test_pages_shapes(name):
    w = synth.make_la_workload(name, device="cuda")
    out, pool = run(w)
    ref_o, ref_s = reference(w)
    check(out, ref_o, f"{name} out", **(PREFILL if w.mode == "prefill" else DECODE_OUT))
    check_states(pool, w, ref_s, name, **(PREFILL if w.mode == "prefill" else DECODE_STATE))
