"""Pins of the FP8 (E4M3) KV-cache oracle path (CPU).

* every one of the 256 E4M3 codes decodes to torch's float8_e4m3fn value
  (library routine) and the format's landmark values;
* attention over E4M3 pools with per-kv-head scales equals brute-force fp64
  softmax attention on the dequantised pools (contiguous copy, explicit mask);
* folding a factor between softmax scale and K scale, or between V scale and
  the output, leaves the result unchanged."""
import math

import numpy as np
import pytest
import torch

import oracle
from segmented_kv_cache_b200 import synth

from test_oracle_pins import brute_force, random_case


def test_all_codes_match_torch_and_landmarks():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2  # 0x7f, 0xff
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x38] == 1.0 and ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9
    assert ours[0x08] == 2.0 ** -6 and ours[0xB8] == -1.0 and ours[0x80] == 0.0


def fp8_case(seed, causal=True, q_mode="chunk"):
    case = random_case(seed, hq=4, hkv=2, d=16, causal=causal, q_mode=q_mode)
    g = torch.Generator().manual_seed(seed + 100)
    hkv = case["k_pool"].shape[1]
    ks = (0.5 + torch.rand(hkv, generator=g, dtype=torch.float64)) / 64
    vs = (0.5 + torch.rand(hkv, generator=g, dtype=torch.float64)) / 64
    kf = torch.nan_to_num(case["k_pool"].float(), nan=0.0) / ks.float().view(1, -1, 1)
    vf = torch.nan_to_num(case["v_pool"].float(), nan=0.0) / vs.float().view(1, -1, 1)
    case["k8"] = kf.clamp(-448, 448).to(torch.float8_e4m3fn)
    case["v8"] = vf.clamp(-448, 448).to(torch.float8_e4m3fn)
    case["ks"], case["vs"] = ks, vs
    return case


def run_fp8(case, **kw):
    return oracle.attention_fp8(case["q_lens"], case["seg_starts"], case["seg_lens"], case["q"],
                                case["k8"], case["v8"], kw.get("ks", case["ks"]),
                                kw.get("vs", case["vs"]), kw.get("scale", case["scale"]),
                                case["causal"])


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_equals_brute_force_on_dequantised_pools(seed, causal):
    case = fp8_case(seed, causal, "chunk" if seed % 2 else "full")
    out, lse = run_fp8(case)
    deq = dict(case, k_pool=case["k8"].double() * case["ks"].view(1, -1, 1),
               v_pool=case["v8"].double() * case["vs"].view(1, -1, 1))
    bo, bl = brute_force(deq)
    torch.testing.assert_close(out, bo, rtol=0, atol=1e-12)
    torch.testing.assert_close(lse, bl, rtol=0, atol=1e-12)


def test_scale_factors_can_move_between_softmax_and_k_and_between_v_and_output():
    case = fp8_case(7)
    out, lse = run_fp8(case)
    out2, lse2 = run_fp8(case, scale=case["scale"] * 4, ks=case["ks"] / 4, vs=case["vs"] * 2)
    torch.testing.assert_close(lse2, lse, rtol=0, atol=1e-12)
    torch.testing.assert_close(out2, out * 2, rtol=0, atol=1e-12)
