"""Randomised GPU parity: shapes, head groupings, dtypes and hooks drawn at random
(seeded), each checked element by element against the fp64 oracle, plus the tile map
bit for bit.  Complements the fixed configurations with ragged and odd combinations."""
import math

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings, strategies as st

import oracle
import synth
from tests.helpers import compare

pytestmark = pytest.mark.gpu

MASKS = ["none", "causal", "sliding_window", "kv_le_q_plus_offset", "causal_fast"]


@settings(max_examples=40, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(Sq=st.integers(1, 700), Skv=st.integers(1, 700), D=st.sampled_from([64, 128]),
       grp=st.sampled_from([(1, 1), (2, 1), (4, 2), (6, 2), (8, 1)]), B=st.integers(1, 2),
       dtype=st.sampled_from(["bf16", "f16"]), mask=st.sampled_from(MASKS),
       alibi=st.booleans(), window=st.integers(1, 300), offset=st.integers(-400, 400),
       sigma=st.sampled_from([0.5, 1.0, 2.0]), seed=st.integers(0, 10_000))
def test_random_forward(Sq, Skv, D, grp, B, dtype, mask, alibi, window, offset, sigma, seed):
    import attention_flex_attn_b200 as fa
    H, Hkv = grp
    q = synth.normal_tensor((B, H, Sq, D), seed * 8 + 1, sigma, dtype)
    k = synth.normal_tensor((B, Hkv, Skv, D), seed * 8 + 2, sigma, dtype)
    v = synth.normal_tensor((B, Hkv, Skv, D), seed * 8 + 3, 1.0, dtype)
    mods = dict(score_mod="alibi" if alibi else "none", mask_mod=mask, window=window, offset=offset)
    scale = 1.0 / math.sqrt(D)
    bm, bn = fa.tile_sizes(D)
    tm = torch.full((-(-Sq // bm) * -(-Skv // bn),), 255, dtype=torch.uint8, device="cuda")
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, tile_map=tm, **mods)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = oracle.fwd(q, k, v, scale=scale, **mods)
    compare(o, lse, ro, rl, f"{mods} Sq={Sq} Skv={Skv} D={D} H={H}/{Hkv} {dtype}")
    ref_map = oracle.tile_map(mask, Sq, Skv, window=window, offset=offset, bm=bm, bn=bn)
    np.testing.assert_array_equal(tm.cpu().numpy().reshape(ref_map.shape), ref_map)


@settings(max_examples=25, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(B=st.integers(1, 4), grp=st.sampled_from([(1, 1), (4, 4), (8, 2), (12, 3), (24, 1), (34, 2)]),
       cap=st.integers(1, 1500), D=st.sampled_from([64, 128]), dtype=st.sampled_from(["bf16", "f16"]),
       with_mask=st.booleans(), p_mask=st.sampled_from([0.0, 0.1, 0.9]), seed=st.integers(0, 10_000))
def test_random_decode(B, grp, cap, D, dtype, with_mask, p_mask, seed):
    import attention_flex_attn_b200 as fa
    H, Hkv = grp
    q = synth.normal_tensor((B, H, 1, D), seed * 8 + 1, 1.0, dtype)
    kc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 2, 1.0, dtype)
    vc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 3, 1.0, dtype)
    lens = synth.kv_lengths(B, cap, seed * 8 + 4, lo=0)
    mask = synth.bernoulli_neg_inf_mask((B, H, 1, cap), p_mask, seed * 8 + 5, dtype) if with_mask else None
    scale = 1.0 / math.sqrt(D)
    o, lse = fa.decode(q.cuda(), kc.cuda(), vc.cuda(), lens.cuda(), scale,
                       mask=None if mask is None else mask.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = oracle.decode(q, kc, vc, lens, scale, mask=mask)
    compare(o, lse, ro, rl, f"decode B={B} H={H}/{Hkv} cap={cap} D={D} {dtype} mask={with_mask}")
