"""Pins of the fp64 oracle against things other than itself (CPU only).

* hand-derived closed-form fixtures (tests/golden/closed_form_cases.json);
* brute force: torch softmax on a contiguous fp64 copy of each request's K/V
  with an explicitly built bottom-right causal mask;
* closed forms: identical V rows, a single visible key, Q = 0, identical K;
* invariances: re-segmenting, moving segments in the pool, MHA replication;
* chunked-prefill consistency (a chunk over prior context equals the same rows
  of a from-scratch prefill), decode = last row of a causal prefill.

What the method computes: exact softmax attention over keys that live in
contiguous segments of a shared slot pool (Flood README, "Introduction" and
"Kernels > Seg-attn"), with chunked prefill (feature list).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from segmented_kv_cache_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


# --------------------------------------------------------------------------- helpers
def random_case(seed, batch=3, hq=4, hkv=2, d=16, causal=True, max_k=70, nseg_max=4,
                q_mode="chunk"):
    g = torch.Generator().manual_seed(seed)
    k_lens = torch.randint(1, max_k + 1, (batch,), generator=g).tolist()
    if q_mode == "full":
        q_lens = list(k_lens)
    elif q_mode == "decode":
        q_lens = [1] * batch
    else:
        q_lens = [int(torch.randint(0, k + 1, (1,), generator=g)) for k in k_lens]
    seg_lens = [synth.split_uniform_cuts(k, int(torch.randint(1, nseg_max + 1, (1,), generator=g)), g)
                for k in k_lens]
    flat = [x for s in seg_lens for x in s]
    slots = sum(flat) + 37
    starts = synth.place_segments(flat, slots, g)
    it = iter(starts)
    seg_starts = [[next(it) for _ in s] for s in seg_lens]
    q = torch.randn(sum(q_lens), hq, d, generator=g).to(torch.bfloat16)
    k = torch.full((slots, hkv, d), float("nan")).to(torch.bfloat16)
    v = torch.full((slots, hkv, d), float("nan")).to(torch.bfloat16)
    for ss, ll in zip(seg_starts, seg_lens):
        for s, l in zip(ss, ll):
            k[s:s + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
            v[s:s + l] = torch.randn(l, hkv, d, generator=g).to(torch.bfloat16)
    return dict(q_lens=q_lens, seg_starts=seg_starts, seg_lens=seg_lens, q=q, k_pool=k, v_pool=v,
                scale=1.0 / math.sqrt(d), causal=causal)


def run_oracle(case, rows=None):
    return oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"], case["q"],
                            case["k_pool"], case["v_pool"], case["scale"], case["causal"], rows=rows)


def brute_force(case):
    """softmax(QK^T*scale + mask)V per request on a contiguous fp64 copy."""
    q_all = case["q"].double()
    kp, vp = case["k_pool"].double(), case["v_pool"].double()
    hq, d = q_all.shape[1], q_all.shape[2]
    G = hq // kp.shape[1]
    outs, lses = [], []
    tok = 0
    for ql, ss, ll in zip(case["q_lens"], case["seg_starts"], case["seg_lens"]):
        idx = torch.cat([torch.arange(s, s + l) for s, l in zip(ss, ll)]) if ll else \
            torch.zeros(0, dtype=torch.long)
        K = kp[idx].repeat_interleave(G, dim=1)  # [k, hq, d]
        V = vp[idx].repeat_interleave(G, dim=1)
        Q = q_all[tok:tok + ql]
        tok += ql
        k_len = idx.numel()
        scores = torch.einsum("qhd,khd->hqk", Q, K) * case["scale"]
        if case["causal"]:
            i = torch.arange(ql).view(-1, 1)
            j = torch.arange(k_len).view(1, -1)
            mask = j <= (k_len - ql) + i
            scores = scores.masked_fill(~mask, float("-inf"))
        if k_len == 0:
            outs.append(torch.zeros(ql, hq, d, dtype=torch.float64))
            lses.append(torch.full((ql, hq), float("-inf"), dtype=torch.float64))
            continue
        p = torch.softmax(scores, dim=-1)
        outs.append(torch.einsum("hqk,khd->qhd", p, V))
        lses.append(torch.logsumexp(scores, dim=-1).transpose(0, 1))
    return torch.cat(outs), torch.cat(lses)


# --------------------------------------------------------------------------- golden
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_closed_form(case):
    S, hkv, d = case["num_slots"], case["kv_heads"], case["head_dim"]
    k = torch.full((S, hkv, d), float("nan"))
    v = torch.full((S, hkv, d), float("nan"))
    for slot, rows in case["k_rows"].items():
        k[int(slot)] = torch.tensor(rows)
    for slot, rows in case["v_rows"].items():
        v[int(slot)] = torch.tensor(rows)
    c = dict(q_lens=case["q_lens"], seg_starts=case["seg_starts"], seg_lens=case["seg_lens"],
             q=torch.tensor(case["q"]).to(torch.bfloat16), k_pool=k.to(torch.bfloat16),
             v_pool=v.to(torch.bfloat16), scale=case["scale"], causal=case["causal"])
    # the fixture values must be exact in bf16
    assert torch.equal(c["q"].double(), torch.tensor(case["q"], dtype=torch.float64))
    out, lse = run_oracle(c)
    torch.testing.assert_close(out, torch.tensor(case["out"], dtype=torch.float64), rtol=0, atol=1e-12)
    torch.testing.assert_close(lse, torch.tensor(case["lse"], dtype=torch.float64), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("causal", [True, False])
def test_brute_force_random(seed, causal):
    case = random_case(seed, causal=causal, q_mode="chunk" if seed % 2 else "full")
    out, lse = run_oracle(case)
    bo, bl = brute_force(case)
    assert not torch.isnan(out).any()
    torch.testing.assert_close(out, bo, rtol=0, atol=1e-12)
    torch.testing.assert_close(lse, bl, rtol=0, atol=1e-12)


def test_brute_force_config1():
    wl = synth.make_workload(1)
    b = wl.batches[0]
    case = dict(q_lens=b.q_lens, seg_starts=b.seg_starts, seg_lens=b.seg_lens, q=b.q,
                k_pool=wl.k_pool, v_pool=wl.v_pool, scale=wl.scale, causal=b.causal)
    out, lse = run_oracle(case)
    bo, bl = brute_force(case)
    torch.testing.assert_close(out, bo, rtol=0, atol=1e-12)
    torch.testing.assert_close(lse, bl, rtol=0, atol=1e-12)


def test_brute_force_config2_sampled_rows():
    wl = synth.make_workload(2)
    b = wl.batches[0]
    case = dict(q_lens=b.q_lens, seg_starts=b.seg_starts, seg_lens=b.seg_lens, q=b.q,
                k_pool=wl.k_pool, v_pool=wl.v_pool, scale=wl.scale, causal=b.causal)
    g = torch.Generator().manual_seed(7)
    toks = torch.cat([torch.tensor([0, 1023]), torch.randint(0, 1024, (30,), generator=g)])
    heads = torch.randint(0, 64, (toks.numel(),), generator=g)
    out, lse = run_oracle(case, rows=(toks.numpy(), heads.numpy()))
    bo, bl = brute_force(case)
    torch.testing.assert_close(out, bo[toks, heads], rtol=0, atol=1e-12)
    torch.testing.assert_close(lse, bl[toks, heads], rtol=0, atol=1e-12)


def test_empty_and_zero_length_requests():
    case = random_case(11, batch=3, causal=False)
    case["q_lens"] = [0, 2, 1]
    case["q"] = case["q"][:3] if case["q"].shape[0] >= 3 else torch.randn(3, 4, 16).to(torch.bfloat16)
    # request 2 has no keys at all: non-causal -> out 0, lse -inf
    case["seg_starts"][2] = []
    case["seg_lens"][2] = []
    out, lse = run_oracle(case)
    assert out.shape[0] == 3
    assert torch.all(out[2] == 0) and torch.all(torch.isneginf(lse[2]))
    bo, bl = brute_force(case)
    torch.testing.assert_close(out, bo, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- closed forms
def test_identical_v_rows_return_that_row():
    case = random_case(21, causal=True)
    v = torch.randn(case["v_pool"].shape[1], case["v_pool"].shape[2]).to(torch.bfloat16)
    case["v_pool"] = v.unsqueeze(0).expand_as(case["v_pool"]).clone()
    out, _ = run_oracle(case)
    G = case["q"].shape[1] // v.shape[0]
    expect = v.double().repeat_interleave(G, dim=0).unsqueeze(0).expand_as(out)
    valid = torch.tensor([True] * out.shape[0])
    torch.testing.assert_close(out[valid], expect[valid], rtol=0, atol=1e-13)


def test_single_visible_key():
    # causal full prefill: query 0 sees only logical key 0
    case = random_case(22, causal=True, q_mode="full")
    out, lse = run_oracle(case)
    kp, vp = case["k_pool"].double(), case["v_pool"].double()
    G = case["q"].shape[1] // kp.shape[1]
    tok = 0
    for ql, ss in zip(case["q_lens"], case["seg_starts"]):
        slot0 = ss[0]
        for h in range(case["q"].shape[1]):
            g = h // G
            torch.testing.assert_close(out[tok, h], vp[slot0, g], rtol=0, atol=0)
            s = case["scale"] * float((case["q"][tok, h].double() * kp[slot0, g]).sum())
            assert abs(float(lse[tok, h]) - s) <= 1e-12
        tok += ql


def test_zero_query_gives_mean_and_log_count():
    case = random_case(23, causal=True, q_mode="chunk")
    case["q"] = torch.zeros_like(case["q"])
    out, lse = run_oracle(case)
    vp = case["v_pool"].double()
    G = case["q"].shape[1] // vp.shape[1]
    tok = 0
    for ql, ss, ll in zip(case["q_lens"], case["seg_starts"], case["seg_lens"]):
        idx = torch.cat([torch.arange(s, s + l) for s, l in zip(ss, ll)])
        k_len = idx.numel()
        for i in range(ql):
            n_vis = (k_len - ql) + i + 1
            mean = vp[idx[:n_vis]].mean(0).repeat_interleave(G, dim=0)
            torch.testing.assert_close(out[tok + i], mean, rtol=0, atol=1e-13)
            assert torch.allclose(lse[tok + i], torch.full_like(lse[tok + i], math.log(n_vis)),
                                  atol=1e-13, rtol=0)
        tok += ql


def test_identical_keys_shift_lse_only():
    case = random_case(24, causal=False, q_mode="chunk")
    krow = torch.randn(case["k_pool"].shape[1], case["k_pool"].shape[2]).to(torch.bfloat16)
    case["k_pool"] = krow.unsqueeze(0).expand_as(case["k_pool"]).clone()
    out, lse = run_oracle(case)
    vp = case["v_pool"].double()
    G = case["q"].shape[1] // vp.shape[1]
    tok = 0
    for ql, ss, ll in zip(case["q_lens"], case["seg_starts"], case["seg_lens"]):
        idx = torch.cat([torch.arange(s, s + l) for s, l in zip(ss, ll)])
        mean = vp[idx].mean(0).repeat_interleave(G, dim=0)
        for i in range(ql):
            torch.testing.assert_close(out[tok + i], mean, rtol=0, atol=1e-13)
            for h in range(case["q"].shape[1]):
                s = case["scale"] * float((case["q"][tok + i, h].double() * krow[h // G].double()).sum())
                assert abs(float(lse[tok + i, h]) - (s + math.log(idx.numel()))) <= 1e-12
        tok += ql


# --------------------------------------------------------------------------- invariances
def test_resegmenting_is_bit_identical():
    case = random_case(31, causal=True, nseg_max=2)
    out, lse = run_oracle(case)
    g = torch.Generator().manual_seed(5)
    new_starts, new_lens = [], []
    for ss, ll in zip(case["seg_starts"], case["seg_lens"]):
        s2, l2 = [], []
        for s, l in zip(ss, ll):
            pieces = synth.split_uniform_cuts(l, 3, g)
            pos = s
            for p in pieces:
                s2.append(pos)
                l2.append(p)
                pos += p
        new_starts.append(s2)
        new_lens.append(l2)
    case2 = dict(case, seg_starts=new_starts, seg_lens=new_lens)
    out2, lse2 = run_oracle(case2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_slot_permutation_is_bit_identical():
    case = random_case(32, causal=True)
    out, lse = run_oracle(case)
    flat = [x for s in case["seg_lens"] for x in s]
    S2 = sum(flat) + 101
    g = torch.Generator().manual_seed(9)
    starts2 = synth.place_segments(flat, S2, g)
    kp2 = torch.full((S2,) + case["k_pool"].shape[1:], float("nan")).to(torch.bfloat16)
    vp2 = kp2.clone()
    it = iter(starts2)
    new_starts = []
    for ss, ll in zip(case["seg_starts"], case["seg_lens"]):
        row = []
        for s, l in zip(ss, ll):
            t = next(it)
            kp2[t:t + l] = case["k_pool"][s:s + l]
            vp2[t:t + l] = case["v_pool"][s:s + l]
            row.append(t)
        new_starts.append(row)
    case2 = dict(case, seg_starts=new_starts, k_pool=kp2, v_pool=vp2)
    out2, lse2 = run_oracle(case2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_mha_replication_matches_gqa_and_grouping_matters():
    case = random_case(33, hq=4, hkv=2, causal=True)
    out, lse = run_oracle(case)
    G = 2
    case_mha = dict(case, k_pool=case["k_pool"].repeat_interleave(G, dim=1).contiguous(),
                    v_pool=case["v_pool"].repeat_interleave(G, dim=1).contiguous())
    out2, lse2 = run_oracle(case_mha)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    # regrouping kv heads (head h -> kv head h % Hkv instead of h // G) changes the answer
    perm = torch.tensor([0, 2, 1, 3])
    case_perm = dict(case, q=case["q"][:, perm].contiguous())
    out3, _ = run_oracle(case_perm)
    assert not torch.allclose(out3[:, perm], out, atol=1e-3)


def test_chunked_prefill_equals_rows_of_full_prefill():
    full = random_case(41, batch=2, causal=True, q_mode="full")
    out_full, lse_full = run_oracle(full)
    # take the last c queries of each request as a chunk over the rest as prior context
    chunks = [5, 17]
    q_parts, rows = [], []
    tok = 0
    for ql, c in zip(full["q_lens"], chunks):
        c = min(c, ql)
        q_parts.append(full["q"][tok + ql - c: tok + ql])
        rows.extend(range(tok + ql - c, tok + ql))
        tok += ql
    chunk = dict(full, q_lens=[min(c, ql) for ql, c in zip(full["q_lens"], chunks)],
                 q=torch.cat(q_parts))
    out_c, lse_c = run_oracle(chunk)
    assert torch.equal(out_c, out_full[rows]) and torch.equal(lse_c, lse_full[rows])


def test_decode_equals_last_row_of_causal_prefill():
    full = random_case(42, batch=3, causal=True, q_mode="full")
    out_full, lse_full = run_oracle(full)
    last = np.cumsum(full["q_lens"]) - 1
    dec = dict(full, q_lens=[1] * 3, q=full["q"][torch.tensor(last)])
    out_d, lse_d = run_oracle(dec)
    assert torch.equal(out_d, out_full[last]) and torch.equal(lse_d, lse_full[last])


def test_rows_entry_matches_full_entry():
    case = random_case(43, causal=True)
    out, lse = run_oracle(case)
    n = out.shape[0]
    toks = np.repeat(np.arange(n), out.shape[1])
    heads = np.tile(np.arange(out.shape[1]), n)
    o2, l2 = run_oracle(case, rows=(toks, heads))
    assert torch.equal(o2.view_as(out), out) and torch.equal(l2.view_as(lse), lse)


def test_free_slots_never_read():
    # NaN-filled free slots: any stray read would poison the output
    case = random_case(44, causal=True)
    out, lse = run_oracle(case)
    assert not torch.isnan(out).any() and not torch.isnan(lse).any()
