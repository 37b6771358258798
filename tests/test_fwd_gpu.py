"""GPU parity of flex_attn_fwd against the fp64 oracle (through the C ABI).

Covers the tiny oracle check, the S=2048 MHA set, the GQA / odd-length / D=64 /
fp16 matrix, cross-attention with fully masked rows, the S=8192 long-context set on
sampled rows, bit-exact tile maps and element masks, and degenerate shapes.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.helpers import compare, gather_rows, sample_rows

pytestmark = pytest.mark.gpu

CASES = {
    "no_mod": dict(score_mod="none", mask_mod="none"),
    "alibi": dict(score_mod="alibi", mask_mod="none"),
    "causal_via_mask": dict(score_mod="none", mask_mod="causal"),
    "causal_fast": dict(score_mod="none", mask_mod="causal_fast"),
}


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _run(q, k, v, scale, rows=None, **mods):
    fa = _fa()
    dev = torch.device("cuda")
    o, lse = fa.fwd(q.to(dev), k.to(dev), v.to(dev), scale=scale, **mods)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    if rows is None:
        ro, rl = oracle.fwd(q, k, v, scale=scale, **mods)
        return compare(o, lse, ro, rl, str(mods))
    ro, rl = oracle.fwd(q, k, v, scale=scale, rows=rows, **mods)
    return compare(gather_rows(o, rows), gather_rows(lse, rows), ro, rl, str(mods))


# ------------------------------------------------------------------ tiny oracle check (B=1, H=4, S=128, D=64)

@pytest.mark.parametrize("case", ["no_mod", "causal_via_mask", "alibi", "sliding_window"])
def test_tiny(case):
    q, k, v = synth.qkv(1, 4, 4, 128, 128, 64, seed=synth.case_seed(0, 1), device="cuda")
    mods = CASES.get(case, dict(score_mod="none", mask_mod="sliding_window", window=32))
    _run(q, k, v, 1.0 / 8.0, **mods)


# ------------------------------------------------------------------ MHA S=2048 (B=2, H=32, D=128)

@pytest.mark.parametrize("case", ["no_mod", "alibi", "sliding_window", "causal_via_mask", "causal_fast"])
def test_mha_2048(case):
    B, H, S, D = 2, 32, 2048, 128
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=synth.case_seed(1, 0), device="cuda")
    mods = CASES.get(case, dict(score_mod="none", mask_mod="sliding_window", window=256))
    rows = sample_rows(B, H, S, 2048, seed=7, must=[(0, 0, 0), (0, 0, 127), (0, 0, 128), (1, 31, 2047),
                                                     (1, 5, 255), (1, 5, 256), (0, 9, 1000), (1, 31, 1792),
                                                     (0, 4, 1023), (0, 4, 1024)])
    _run(q, k, v, 1.0 / math.sqrt(D), rows=rows, **mods)


# ------------------------------------------------------------------ GQA / odd lengths / D=64 / fp16

GQA_CASES = ["no_mod", "alibi", "causal_via_mask", "sliding_window", "causal_fast"]


@pytest.mark.parametrize("S", [250, 384, 1024, 4096])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_gqa_odd(S, D, dtype):
    B, H, Hkv = 2, 32, 8
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=synth.case_seed(2, S % 97 + D), dtype=dtype, device="cuda")
    n = 2048 if S <= 384 else 256
    rows = sample_rows(B, H, S, n, seed=S + D, must=[(0, 0, 0), (1, 31, S - 1), (0, 3, 127), (0, 3, 128),
                                                     (1, 8, S // 2)])
    for case in GQA_CASES:
        mods = CASES.get(case, dict(score_mod="none", mask_mod="sliding_window", window=256))
        _run(q, k, v, 1.0 / math.sqrt(D), rows=rows, **mods)


# ------------------------------------------------------------------ cross attention

def test_cross_attention_fully_masked():
    """Sq=250, Skv=1024, keep kv <= q - 300: every row fully masked -> O = +0, LSE = -inf."""
    B, H, Hkv, D = 2, 32, 8, 128
    q = synth.normal_tensor((B, H, 250, D), 901)
    k = synth.normal_tensor((B, Hkv, 1024, D), 902)
    v = synth.normal_tensor((B, Hkv, 1024, D), 903)
    fa = _fa()
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), mask_mod="kv_le_q_plus_offset", offset=-300)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and not torch.any(torch.signbit(o.float()))
    assert torch.all(torch.isneginf(lse))
    _run(q, k, v, 1.0 / math.sqrt(D), mask_mod="kv_le_q_plus_offset", offset=-300)


@pytest.mark.parametrize("mods", [dict(), dict(score_mod="alibi"),
                                  dict(mask_mod="kv_le_q_plus_offset", offset=500),
                                  dict(mask_mod="kv_le_q_plus_offset", offset=-100),
                                  dict(mask_mod="causal")])
def test_cross_attention(mods):
    B, H, Hkv, D = 2, 32, 8, 128
    q = synth.normal_tensor((B, H, 250, D), 911)
    k = synth.normal_tensor((B, Hkv, 1024, D), 912)
    v = synth.normal_tensor((B, Hkv, 1024, D), 913)
    _run(q, k, v, 1.0 / math.sqrt(D), **mods)


# ------------------------------------------------------------------ long context S=8192 (sampled rows)

@pytest.mark.parametrize("case", ["no_mod", "alibi", "sliding_window", "causal_via_mask", "causal_fast"])
def test_long_8192(case):
    B, H, S, D = 2, 32, 8192, 128
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=synth.case_seed(4, 0), sigma=0.5, device="cuda")
    mods = CASES.get(case, dict(score_mod="none", mask_mod="sliding_window", window=1024))
    # 2048 seeded rows plus rows 0, 127, 128, 8191, the window edges (1023/1024/1025 for
    # W = 1024), and the first and last rows of the first and last query-tile pairs
    rows = sample_rows(B, H, S, 2048, seed=44, must=[(0, 0, 0), (0, 0, 127), (0, 0, 128), (0, 0, 255),
                                                     (0, 0, 256), (1, 31, 8191), (1, 31, 7936), (1, 31, 8064),
                                                     (0, 17, 1023), (0, 17, 1024), (0, 17, 1025),
                                                     (1, 2, 4095), (1, 2, 4096)])
    _run(q, k, v, 1.0 / math.sqrt(D), rows=rows, **mods)


# ------------------------------------------------------------------ persistent kernel, split last round

# Units (B*H*ceil(ceil(Sq/128)/2)) chosen so that on a 148-SM B200 the persistent kernel
# splits the last round's units into 4, 3 or 2 parts (R = units mod 148 of them), with
# windows that leave some parts empty, a ragged last query tile, a lone query tile in the
# last pair, GQA, alibi and a key length unequal to the query length.  On another SM
# count the split differs, and the oracle comparison holds all the same.
SPLIT_CASES = [
    (1, 38, 38, 1024, 1024, 128, dict()),                                        # R=4, 4 parts
    (1, 49, 7, 1024, 1024, 128, dict(score_mod="alibi")),                        # R=48, 3 parts
    (2, 32, 32, 2048, 2048, 128, dict()),                                        # R=68, 2 parts
    (1, 38, 38, 1024, 1024, 64, dict(mask_mod="sliding_window", window=64)),      # empty parts
    (1, 50, 10, 600, 600, 128, dict(mask_mod="sliding_window", window=200)),      # lone tile
    (1, 40, 8, 1000, 1700, 64, dict(score_mod="alibi")),                         # ragged, Skv != Sq
]


@pytest.mark.parametrize("case", range(len(SPLIT_CASES)))
def test_persistent_split_last_round(case):
    B, H, Hkv, Sq, Skv, D, mods = SPLIT_CASES[case]
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=synth.case_seed(6, case), device="cuda")
    last = [(b, h, i) for b in range(B) for h in (0, H - 1) for i in (0, 127, 128, Sq - 129, Sq - 128, Sq - 1)]
    rows = sample_rows(B, H, Sq, 2048, seed=60 + case, must=last)
    _run(q, k, v, 1.0 / math.sqrt(D), rows=rows, **mods)
    # the merge reads every part from memory in part order, whichever CTA merges: repeat
    # calls agree bit for bit
    fa = _fa()
    o1, l1 = fa.fwd(q, k, v, **mods)
    o2, l2 = fa.fwd(q, k, v, **mods)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_split_two_streams_and_graph_replay():
    """Split launches on two streams at once each use their own workspace; a captured
    graph, which replays the same counter tag, resets the counters after every merge.
    Every result equals the eager single-stream result bit for bit."""
    fa = _fa()
    B, H, Hkv, Sq, Skv, D, mods = SPLIT_CASES[0]
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=synth.case_seed(6, 0), device="cuda")
    o_ref, l_ref = fa.fwd(q, k, v, **mods)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            outs.append(fa.fwd(q, k, v, **mods))
        with torch.cuda.stream(s2):
            outs.append(fa.fwd(q, k, v, **mods))
    torch.cuda.synchronize()
    for o, l in outs:
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
    g_stream = torch.cuda.Stream()
    with torch.cuda.stream(g_stream):
        fa.fwd(q, k, v, **mods)  # creates this stream's workspace before the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=g_stream):
        o_g, l_g = fa.fwd(q, k, v, **mods)
    for _ in range(3):
        o_g.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o_g, o_ref) and torch.equal(l_g, l_ref)
    assert fa.device_status() == 0


# ------------------------------------------------------------------ degenerate shapes

@pytest.mark.parametrize("Sq,Skv", [(1, 1), (1, 300), (7, 1), (129, 129), (130, 5), (255, 513), (512, 128)])
@pytest.mark.parametrize("case", ["no_mod", "causal_via_mask", "alibi"])
def test_degenerate_shapes(Sq, Skv, case):
    q = synth.normal_tensor((1, 4, Sq, 128), 70 + Sq)
    k = synth.normal_tensor((1, 2, Skv, 128), 71 + Skv)
    v = synth.normal_tensor((1, 2, Skv, 128), 72 + Skv)
    _run(q, k, v, 0.09, **CASES[case])


def test_window_of_one_and_lse_none():
    q, k, v = synth.qkv(1, 2, 2, 300, 300, 64, seed=81)
    _run(q, k, v, 0.125, mask_mod="sliding_window", window=1)
    fa = _fa()
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), return_lse=False)
    assert lse is None
    ro, _ = oracle.fwd(q, k, v)
    assert np.abs(o.float().cpu().numpy() - ro).max() < 2e-2


# ------------------------------------------------------------------ bit-exact tile maps and masks

MAP_SHAPES = [(384, 384), (250, 250), (1000, 1000), (250, 1024), (2048, 2048), (640, 640), (129, 700)]
MAP_MODS = [("none", 0, 0), ("causal", 0, 0), ("sliding_window", 256, 0), ("sliding_window", 32, 0),
            ("kv_le_q_plus_offset", 0, -300), ("kv_le_q_plus_offset", 0, 500), ("causal_fast", 0, 0)]


@pytest.mark.parametrize("Sq,Skv", MAP_SHAPES)
@pytest.mark.parametrize("mask,window,offset", MAP_MODS)
def test_tile_map_bit_exact(Sq, Skv, mask, window, offset):
    fa = _fa()
    bm, bn = fa.tile_sizes(64)
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    tm = torch.full((nq * nk,), 255, dtype=torch.uint8, device="cuda")
    q = synth.normal_tensor((1, 1, Sq, 64), 1)
    k = synth.normal_tensor((1, 1, Skv, 64), 2)
    fa.fwd(q.cuda(), k.cuda(), k.cuda(), mask_mod=mask, window=window, offset=offset, tile_map=tm)
    torch.cuda.synchronize()
    ref = oracle.tile_map(mask, Sq, Skv, window=window, offset=offset, bm=bm, bn=bn)
    np.testing.assert_array_equal(tm.cpu().numpy().reshape(nq, nk), ref)


@pytest.mark.parametrize("Sq,Skv", MAP_SHAPES)
@pytest.mark.parametrize("mask,window,offset", MAP_MODS)
def test_mask_eval_bit_exact(Sq, Skv, mask, window, offset):
    fa = _fa()
    keep = fa.mask_eval(mask, Sq, Skv, window=window, offset=offset)
    torch.cuda.synchronize()
    ref = oracle.mask_matrix(mask, Sq, Skv, window=window, offset=offset)
    np.testing.assert_array_equal(keep.cpu().numpy(), ref)
