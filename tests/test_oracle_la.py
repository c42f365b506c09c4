"""Pins of the linear-attention (simple GLA) oracle, on the CPU.

The oracle runs the recurrence token by token.  It is pinned against forms of
the same quantity that share none of its steps: the parallel (attention-like)
closed form evaluated with torch fp64 matrix products, the no-decay cumulative
sum of outer products, the full-reset limit, splitting a request into two calls
through the state, and decode as the last row of a prefill.  Every planted
mistake (ORACLE_MUTANT 8-12) must fail at least one pin."""
import math

import pytest
import torch

import oracle

D = 8
H = 2


def case(seed, q_lens, with_state=True, g_scale=0.3):
    g = torch.Generator().manual_seed(seed)
    T = sum(q_lens)
    q = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(T, H, D, generator=g).to(torch.bfloat16)
    gate = -torch.rand(T, H, generator=g, dtype=torch.float64) * g_scale
    states = torch.randn(len(q_lens) + 1, H, D, D, generator=g, dtype=torch.float64)
    in_slot = [(r + 1) % (len(q_lens) + 1) if with_state and r % 2 == 0 else -1
               for r in range(len(q_lens))]
    return q, k, v, gate, states, in_slot


def closed_form(q_lens, q, k, v, gate, states, in_slot, scale):
    """o = scale (tril(Q K^T . exp(G_t - G_s)) V + exp(G_t) Q S0);
    S_T = exp(G_T) S0 + (K . exp(G_T - G_s))^T V, with G the running sum of g."""
    outs, finals = [], []
    off = 0
    for r, n in enumerate(q_lens):
        o_r = torch.zeros(n, H, D, dtype=torch.float64)
        f_r = torch.zeros(H, D, D, dtype=torch.float64)
        for h in range(H):
            Q = q[off:off + n, h].double()
            K = k[off:off + n, h].double()
            V = v[off:off + n, h].double()
            S0 = states[in_slot[r], h] if in_slot[r] >= 0 else torch.zeros(D, D, dtype=torch.float64)
            G = torch.cumsum(gate[off:off + n, h], 0)
            decay = torch.tril(torch.exp(G[:, None] - G[None, :]))
            o_r[:, h] = scale * ((Q @ K.T * decay) @ V + torch.exp(G)[:, None] * (Q @ S0))
            GT = G[-1] if n else torch.tensor(0.0, dtype=torch.float64)
            f_r[h] = torch.exp(GT) * S0 + (K * torch.exp(GT - G)[:, None]).T @ V
        outs.append(o_r)
        finals.append(f_r)
        off += n
    return torch.cat(outs), torch.stack(finals)


def rel_err(a, b):
    return float((a - b).abs().max() / b.abs().max().clamp(min=1e-30))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_parallel_closed_form(seed):
    q_lens = [5, 0, 17, 1]
    q, k, v, gate, states, slots = case(seed, q_lens)
    scale = 1 / math.sqrt(D)
    o, s = oracle.linear_attention(q_lens, q, k, v, gate, scale, states, slots)
    ro, rs = closed_form(q_lens, q, k, v, gate, states, slots, scale)
    assert rel_err(o, ro) < 1e-12 and rel_err(s, rs) < 1e-12


def test_no_decay_is_cumulative_outer_products():
    q_lens = [9]
    q, k, v, gate, states, _ = case(3, q_lens)
    o, s = oracle.linear_attention(q_lens, q, k, v, torch.zeros_like(gate), 0.5)
    outer = torch.einsum("thi,thj->thij", k.double(), v.double())
    S = torch.cumsum(outer, 0)
    ref = 0.5 * torch.einsum("thi,thij->thj", q.double(), S)
    assert rel_err(o, ref) < 1e-12 and rel_err(s[0], S[-1]) < 1e-12


def test_full_reset_limit():
    # exp(-60) < 1e-26: the state keeps only the current token
    q_lens = [6]
    q, k, v, gate, states, _ = case(4, q_lens)
    o, s = oracle.linear_attention(q_lens, q, k, v, torch.full_like(gate, -60.0), 1.0,
                                   states, [0])
    ref = torch.einsum("thi,thi->th", q.double(), k.double())[..., None] * v.double()
    assert rel_err(o, ref) < 1e-12
    assert rel_err(s[0], torch.einsum("hi,hj->hij", k[-1].double(), v[-1].double())) < 1e-12


def test_split_through_the_state_equals_one_call():
    q_lens = [20]
    q, k, v, gate, states, _ = case(5, q_lens)
    o, s = oracle.linear_attention(q_lens, q, k, v, gate, 0.3, states, [1])
    o1, s1 = oracle.linear_attention([7], q[:7], k[:7], v[:7], gate[:7], 0.3, states, [1])
    o2, s2 = oracle.linear_attention([13], q[7:], k[7:], v[7:], gate[7:], 0.3, s1, [0])
    assert rel_err(torch.cat([o1, o2]), o) < 1e-12 and rel_err(s2, s) < 1e-12


def test_decode_is_last_prefill_row():
    q_lens = [11]
    q, k, v, gate, states, _ = case(6, q_lens)
    o, s = oracle.linear_attention(q_lens, q, k, v, gate, 0.3, states, [1])
    _, s10 = oracle.linear_attention([10], q[:10], k[:10], v[:10], gate[:10], 0.3, states, [1])
    od, sd = oracle.linear_attention([1], q[10:], k[10:], v[10:], gate[10:], 0.3, s10, [0])
    assert rel_err(od[0], o[-1]) < 1e-12 and rel_err(sd, s) < 1e-12


@pytest.mark.parametrize("mutant", [8, 9, 10, 11, 12])
def test_planted_mistakes_are_caught(mutant):
    oracle.build(mutant=mutant)
    q_lens = [5, 0, 17, 1]
    q, k, v, gate, states, slots = case(0, q_lens)
    scale = 1 / math.sqrt(D)
    o, s = oracle.linear_attention(q_lens, q, k, v, gate, scale, states, slots, mutant=mutant)
    ro, rs = closed_form(q_lens, q, k, v, gate, states, slots, scale)
    assert rel_err(o, ro) > 1e-3 or rel_err(s, rs) > 1e-3
