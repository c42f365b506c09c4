"""Each planted oracle mistake (a dropped term, a wrong index, a swapped operand,
a wrong mask alignment) must fail at least one of the pins that the real oracle
passes.  The mistakes live in the oracle's C source behind ORACLE_MUTANT and are
compiled here, on the CPU, into separate libraries."""
import json
import math

import numpy as np
import pytest
import torch

import oracle
from segmented_kv_cache_b200 import synth

from test_oracle_pins import GOLDEN, brute_force, random_case

MUTANTS = {1: "no scale", 2: "top-left causal", 3: "kv head h % Hkv", 4: "slot-order walk",
           5: "lse without max", 6: "no 1/l", 7: "K instead of V"}


def _run(case, mutant, rows=None):
    return oracle.attention(case["q_lens"], case["seg_starts"], case["seg_lens"], case["q"],
                            case["k_pool"], case["v_pool"], case["scale"], case["causal"],
                            rows=rows, mutant=mutant)


def _close(a, b, tol=1e-9):
    fin = torch.isfinite(b)
    return torch.equal(torch.isfinite(a), fin) and bool((a[fin] - b[fin]).abs().max() <= tol) \
        if fin.any() else torch.equal(torch.isfinite(a), fin)


def pins_pass(mutant):
    """The pins as booleans (the assertions live in test_oracle_pins)."""
    # golden closed forms
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        S, hkv, d = c["num_slots"], c["kv_heads"], c["head_dim"]
        k = torch.full((S, hkv, d), float("nan"))
        v = torch.full((S, hkv, d), float("nan"))
        for slot, rows in c["k_rows"].items():
            k[int(slot)] = torch.tensor(rows)
        for slot, rows in c["v_rows"].items():
            v[int(slot)] = torch.tensor(rows)
        case = dict(q_lens=c["q_lens"], seg_starts=c["seg_starts"], seg_lens=c["seg_lens"],
                    q=torch.tensor(c["q"]).to(torch.bfloat16), k_pool=k.to(torch.bfloat16),
                    v_pool=v.to(torch.bfloat16), scale=c["scale"], causal=c["causal"])
        o, l = _run(case, mutant)
        if not (_close(o, torch.tensor(c["out"], dtype=torch.float64), 1e-12) and
                _close(l, torch.tensor(c["lse"], dtype=torch.float64), 1e-12)):
            return False
    # brute force on random chunked / full cases, causal and not, with GQA
    for seed in range(3):
        for causal in (True, False):
            case = random_case(200 + seed, hq=4, hkv=2, causal=causal,
                               q_mode="chunk" if seed % 2 else "full")
            o, l = _run(case, mutant)
            bo, bl = brute_force(case)
            if not (_close(o, bo, 1e-12) and _close(l, bl, 1e-12)):
                return False
    return True


def test_real_oracle_passes_the_pins():
    assert pins_pass(0)


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_planted_mistake_is_caught(mutant):
    assert not pins_pass(mutant), f"pins did not catch: {MUTANTS[mutant]}"
