"""Pins for the oracle's e4m3 (fp8) path.

FP8 flex paths are named as a later phase on FlyDSL PR 931 "Add flex_attention (score_mod
/ mask_mod) on the generic flash-attention kernel" (Out of scope: "gfx950 dualwave/fp8
flex paths"). The oracle decodes e4m3 codes exactly and applies per-tensor descales; the
decode is checked code by code against torch's float8_e4m3fn conversion (a library
special case), and the forward against the 16-bit path on the same values (every e4m3
value is exact in bf16), with power-of-two descales folded in exactly.
"""
import numpy as np
import torch

import synth


def test_e4m3_decode_matches_torch(oracle_mod):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def _fp8_inputs(B, H, Hkv, Sq, Skv, D, seed):
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=seed)
    return tuple(t.float().to(torch.float8_e4m3fn) for t in (q, k, v))


def test_fp8_forward_equals_bf16_path_on_same_values(oracle_mod):
    q8, k8, v8 = _fp8_inputs(1, 4, 2, 37, 53, 16, seed=95)
    for mods in (dict(), dict(mask_mod="causal", score_mod="alibi"), dict(mask_mod="sliding_window", window=9)):
        o8, l8 = oracle_mod.fwd_fp8(q8, k8, v8, scale=0.3, **mods)
        ob, lb = oracle_mod.fwd(q8.to(torch.bfloat16), k8.to(torch.bfloat16), v8.to(torch.bfloat16), scale=0.3, **mods)
        np.testing.assert_array_equal(o8, ob)
        np.testing.assert_array_equal(l8, lb)


def test_fp8_descales_fold_exactly(oracle_mod):
    q8, k8, v8 = _fp8_inputs(2, 2, 2, 20, 30, 16, seed=96)
    o8, l8 = oracle_mod.fwd_fp8(q8, k8, v8, descale_q=2.0, descale_k=0.5, descale_v=4.0, scale=0.25,
                                mask_mod="causal")
    bf = lambda t, c: (t.double() * c).to(torch.bfloat16)
    ob, lb = oracle_mod.fwd(bf(q8, 2.0), bf(k8, 0.5), bf(v8, 4.0), scale=0.25, mask_mod="causal")
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)
