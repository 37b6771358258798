"""GPU parity of flex_attn_fwd_block_sparse (BlockMask) against the fp64 oracle.

Block sparsity is named as the next phase on FlyDSL PR 931 "Add flex_attention
(score_mod / mask_mod) on the generic flash-attention kernel" (Out of scope); the lists
follow PyTorch's BlockMask convention (partial blocks apply mask_mod, full blocks only
kv_idx < Skv, unlisted blocks are dropped).

Covers: random lists with repeated / out-of-range indices and over-long counts on shapes
with several tiles and ragged tails (D 64/128, bf16/f16, every mask_mod, alibi, GQA,
broadcast batch/head lists); lists read off the analytic tile map reproduce
flex_attn_fwd bit for bit; all-full lists reproduce the unmasked kernel bit for bit; the
empty mask; the debug tile map of what the kernel visited; S=8192 on sampled rows.
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.helpers import compare, gather_rows, random_block_lists, sample_rows

pytestmark = pytest.mark.gpu

BLOCK = 128


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _dev(*arrays):
    return [None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to("cuda") for a in arrays]


def _run_blocks(q, k, v, lists, scale, tile_map=None, **mods):
    fa = _fa()
    kn, ki, fn, fi = _dev(*lists)
    o, lse = fa.fwd_block_sparse(q.cuda(), k.cuda(), v.cuda(), kn, ki, fn, fi, scale=scale, tile_map=tile_map,
                                 **mods)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return o, lse


MODS = [
    dict(score_mod="none", mask_mod="none"),
    dict(score_mod="none", mask_mod="causal"),
    dict(score_mod="alibi", mask_mod="causal"),
    dict(score_mod="alibi", mask_mod="none"),
    dict(score_mod="none", mask_mod="sliding_window", window=200),
    dict(score_mod="none", mask_mod="kv_le_q_plus_offset", offset=-150),
]


@pytest.mark.parametrize("mods", MODS, ids=lambda m: "-".join(str(x) for x in m.values()))
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f16"), (128, "f16"), (64, "bf16")])
@pytest.mark.parametrize("bcast", ["per_head", "shared", "per_head_only"])
def test_random_lists(mods, D, dtype, bcast):
    B, H, Hkv, Sq, Skv = 2, 4, 2, 300, 700
    nq, nk = -(-Sq // BLOCK), -(-Skv // BLOCK)
    Bm, Hm = {"per_head": (B, H), "shared": (1, 1), "per_head_only": (1, H)}[bcast]
    rng = np.random.default_rng(zlib.crc32(repr((D, dtype, bcast, mods)).encode()))
    lists = random_block_lists(rng, Bm, Hm, nq, nk, max_blocks=nk + 2, p_full=0.35, p_part=0.45)
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=synth.case_seed(40, D), dtype=dtype)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run_blocks(q, k, v, lists, scale, **mods)
    ro, rl = oracle.fwd_block_sparse(q, k, v, *lists, scale=scale, **mods)
    compare(o, lse, ro, rl, f"{mods} {bcast}")


@pytest.mark.parametrize("mask,window,offset", [("causal", 0, 0), ("sliding_window", 300, 0),
                                                ("kv_le_q_plus_offset", 0, 200), ("none", 0, 0)])
@pytest.mark.parametrize("Sq,Skv", [(1000, 1000), (640, 1300)])
def test_tile_map_lists_bit_exact_with_analytic(mask, window, offset, Sq, Skv):
    """Lists naming exactly the tiles the mask_mod range visits give the same kernel work
    in the same order as flex_attn_fwd, hence identical bits."""
    fa = _fa()
    B, H, D = 2, 4, 128
    q, k, v = synth.qkv(B, H, 2, Sq, Skv, D, seed=synth.case_seed(41, Sq), device="cuda")
    mods = dict(score_mod="alibi", mask_mod=mask, window=window, offset=offset)
    tm = oracle.tile_map(mask, Sq, Skv, window, offset)
    lists = oracle.block_mask_from_tile_map(tm, 1, 1)
    o_b, l_b = _run_blocks(q, k, v, lists, 0.09, **mods)
    o_a, l_a = fa.fwd(q, k, v, scale=0.09, **mods)
    torch.cuda.synchronize()
    assert torch.equal(o_b, o_a)
    assert torch.equal(l_b, l_a)
    # the same tiles listed as partial only: reclassified on the device, same bits again
    kn, ki, fn, fi = lists
    nk = tm.shape[1]
    part_n = (kn + fn).astype(np.int32)
    part_i = np.zeros((1, 1, tm.shape[0], nk), np.int32)
    for t in range(tm.shape[0]):
        us = [u for u in range(nk) if tm[t, u] != 0]
        part_i[0, 0, t, :len(us)] = us
    o_p, l_p = _run_blocks(q, k, v, (part_n, part_i, None, None), 0.09, **mods)
    assert torch.equal(o_p, o_a)
    assert torch.equal(l_p, l_a)


@pytest.mark.parametrize("Skv", [1024, 1000])
def test_all_full_bit_exact_with_unmasked(Skv):
    fa = _fa()
    B, H, Sq, D = 1, 8, 512, 128
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=synth.case_seed(42, Skv), device="cuda")
    nq, nk = -(-Sq // BLOCK), -(-Skv // BLOCK)
    fn = np.full((1, 1, nq), nk, np.int32)
    fi = np.broadcast_to(np.arange(nk, dtype=np.int32)[::-1], (1, 1, nq, nk)).copy()
    # mask_mod is ignored on full blocks
    o_b, l_b = _run_blocks(q, k, v, (None, None, fn, fi), 0.1, mask_mod="causal")
    o_a, l_a = fa.fwd(q, k, v, scale=0.1)
    torch.cuda.synchronize()
    assert torch.equal(o_b, o_a)
    assert torch.equal(l_b, l_a)


def test_empty_and_unusable_lists():
    """Counts of 0, negative counts and lists of out-of-range indices only: every row
    is fully masked (O = +0, LSE = -inf)."""
    B, H, Sq, Skv, D = 1, 2, 260, 300, 64
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=3)
    nq, nk = -(-Sq // BLOCK), -(-Skv // BLOCK)
    kn = np.array([[[0, -4, 2]]], np.int32).repeat(H, 1)
    ki = np.array([[[[0, 1], [1, 2], [-1, nk]]]], np.int32).repeat(H, 1)
    o, lse = _run_blocks(q, k, v, (kn, ki, None, None), 0.125)
    assert torch.all(o == 0) and not torch.any(torch.signbit(o.float()))
    assert torch.all(torch.isneginf(lse))


def _expected_map(lists, mask, Sq, Skv, window, offset):
    kn, ki, fn, fi = lists
    nq, nk = -(-Sq // BLOCK), -(-Skv // BLOCK)
    tm = oracle.tile_map(mask, Sq, Skv, window, offset)
    exp = np.zeros((nq, nk), np.uint8)

    def named(num, idx, t):
        if num is None:
            return set()
        c = max(0, min(int(num[0, 0, t]), idx.shape[-1]))
        return {int(u) for u in idx[0, 0, t, :c] if 0 <= u < nk}
    for t in range(nq):
        full, part = named(fn, fi, t), named(kn, ki, t)
        for u in range(nk):
            if u in full:
                exp[t, u] = 2 if (u + 1) * BLOCK > Skv else 1
            elif u in part:
                exp[t, u] = tm[t, u]
    return exp


@pytest.mark.parametrize("mask,window,offset", [("causal", 0, 0), ("sliding_window", 260, 0), ("none", 0, 0)])
def test_tile_map_of_visited_tiles(mask, window, offset):
    B, H, Sq, Skv, D = 1, 2, 900, 1100, 128
    nq, nk = -(-Sq // BLOCK), -(-Skv // BLOCK)
    rng = np.random.default_rng(11 + window)
    lists = random_block_lists(rng, 1, 1, nq, nk, max_blocks=nk + 1)
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=12)
    tmap = torch.full((nq * nk,), 77, dtype=torch.uint8, device="cuda")
    o, lse = _run_blocks(q, k, v, lists, 0.1, tile_map=tmap, mask_mod=mask, window=window, offset=offset)
    got = tmap.cpu().numpy().reshape(nq, nk)
    np.testing.assert_array_equal(got, _expected_map(lists, mask, Sq, Skv, window, offset))
    ro, rl = oracle.fwd_block_sparse(q, k, v, *lists, scale=0.1, mask_mod=mask, window=window, offset=offset)
    compare(o, lse, ro, rl, mask)


@pytest.mark.parametrize("density,mods", [(0.5, dict(mask_mod="causal")), (0.25, dict(score_mod="alibi")),
                                          (0.5, dict(mask_mod="sliding_window", window=1024))])
def test_long_8192_sampled(density, mods):
    """B=2, H=32, S=8192, D=128 with random per-head lists; sampled rows vs the oracle."""
    B, H, S, D = 2, 32, 8192, 128
    nq = nk = S // BLOCK
    rng = np.random.default_rng(int(density * 100) + len(mods))
    full = rng.random((B, H, nq, nk)) < density * 0.5
    part = (rng.random((B, H, nq, nk)) < density) & ~full
    def to_lists(sel):
        num = sel.sum(-1).astype(np.int32)
        idx = np.zeros((B, H, nq, nk), np.int32)
        order = np.argsort(~sel, axis=-1, kind="stable")   # selected blocks first, ascending
        idx[...] = order
        return num, idx
    kn, ki = to_lists(part)
    fn, fi = to_lists(full)
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=synth.case_seed(43, int(density * 10)), device="cuda")
    scale = 1.0 / math.sqrt(D)
    o, lse = _run_blocks(q, k, v, (kn, ki, fn, fi), scale, **mods)
    rows = sample_rows(B, H, S, 192, seed=5, must=[(0, 0, 0), (1, 31, S - 1), (0, 7, 4095), (1, 2, 128)])
    ro, rl = oracle.fwd_block_sparse(q.cpu(), k.cpu(), v.cpu(), kn, ki, fn, fi, scale=scale, rows=rows, **mods)
    compare(gather_rows(o, rows), gather_rows(lse, rows), ro, rl, str(mods))
