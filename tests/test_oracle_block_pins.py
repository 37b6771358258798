"""Pins for the oracle's block-sparse forward (BlockMask).

Block sparsity is named on FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod) on
the generic flash-attention kernel" (Out of scope: the next phase) without a definition;
the oracle takes PyTorch's BlockMask convention (per query tile, a list of partial key
blocks that still apply mask_mod and a list of full key blocks that do not).

The pins check the oracle against things other than its own loop:
  * a dense torch float64 softmax whose keep matrix the test builds from Python sets of
    block indices (duplicates, out-of-range entries and over-long counts included),
  * identities that reduce the block mask to already pinned routines (every block
    partial == the analytic mask_mod; every block full == no mask; the lists read off an
    analytic tile map == that mask_mod),
  * the empty mask (every row 0 / -inf) and numpy broadcasting of [1, 1, ...] lists.
"""
import numpy as np
import pytest
import torch

import synth
from tests.helpers import random_block_lists as _random_lists

TOL = 1e-12


def _sets(num, idx, t_row, nk):
    """Block indices a (clamped) list names for one query-tile row."""
    if num is None:
        return set()
    cnt = int(num[t_row])
    cnt = max(0, min(cnt, idx.shape[-1]))
    return {int(u) for u in idx[t_row][:cnt] if 0 <= int(u) < nk}


def _dense_keep(elem_keep, kn, ki, fn, fi, B, H, Sq, Skv, bm, bn):
    """[B, H, Sq, Skv] keep matrix from the lists, built block by block."""
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    keep = np.zeros((B, H, Sq, Skv), dtype=bool)
    for b in range(B):
        for h in range(H):
            for t in range(nq):
                full = _sets(None if fn is None else fn.reshape(B, H, nq)[b, h],
                             None if fi is None else fi.reshape(B, H, nq, -1)[b, h], t, nk)
                part = _sets(None if kn is None else kn.reshape(B, H, nq)[b, h],
                             None if ki is None else ki.reshape(B, H, nq, -1)[b, h], t, nk) - full
                rs = slice(t * bm, min((t + 1) * bm, Sq))
                for u in full:
                    keep[b, h, rs, u * bn:min((u + 1) * bn, Skv)] = True
                for u in part:
                    cs = slice(u * bn, min((u + 1) * bn, Skv))
                    keep[b, h, rs, cs] = elem_keep[rs, cs]
    return keep


def _torch_masked(q, k, v, keep, scale, alibi=False):
    B, H, Sq, D = q.shape
    Hkv = k.shape[1]
    kk = k.double().repeat_interleave(H // Hkv, dim=1)
    vv = v.double().repeat_interleave(H // Hkv, dim=1)
    s = torch.einsum("bhid,bhjd->bhij", q.double(), kk) * scale
    if alibi:
        Skv = k.shape[2]
        slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float64)
        rel = torch.arange(Skv, dtype=torch.float64)[None, :] - torch.arange(Sq, dtype=torch.float64)[:, None]
        s = s + slopes[:, None, None] * rel
    kt = torch.from_numpy(keep)
    s = s.masked_fill(~kt, float("-inf"))
    any_row = kt.any(-1)
    p = torch.softmax(s.masked_fill(~any_row[..., None], 0.0), -1) * any_row[..., None]
    o = p @ vv
    lse = torch.logsumexp(s, -1)
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("mask,window,offset,score", [
    ("none", 0, 0, "none"), ("causal", 0, 0, "none"), ("sliding_window", 6, 0, "alibi"),
    ("kv_le_q_plus_offset", 0, -5, "none"), ("causal", 0, 0, "alibi")])
def test_block_sparse_equals_dense_masked_softmax(oracle_mod, mask, window, offset, score):
    """Random partial / full lists (duplicates, bad indices, over-long and negative
    counts) == torch float64 softmax with the keep matrix the lists describe."""
    B, H, Hkv, Sq, Skv, D, bm, bn = 2, 4, 2, 23, 37, 8, 4, 8
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    rng = np.random.default_rng(1234 + len(mask) + offset)
    kn, ki, fn, fi = _random_lists(rng, B, H, nq, nk, max_blocks=nk + 1)
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=77)
    scale = 0.41
    o, lse = oracle_mod.fwd_block_sparse(q, k, v, kn, ki, fn, fi, scale=scale, score_mod=score,
                                         mask_mod=mask, window=window, offset=offset, bm=bm, bn=bn)
    elem = oracle_mod.mask_matrix(mask, Sq, Skv, window, offset).astype(bool)
    keep = _dense_keep(elem, kn, ki, fn, fi, B, H, Sq, Skv, bm, bn)
    assert keep.any() and not keep.all(-1).all()
    ref_o, ref_lse = _torch_masked(q, k, v, keep, scale, alibi=score == "alibi")
    np.testing.assert_allclose(o, ref_o, atol=TOL, rtol=0)
    empty = ~keep.any(-1)
    assert np.all(np.isneginf(lse[empty])) and np.all(o[empty] == 0.0)
    np.testing.assert_allclose(lse[~empty], ref_lse[~empty], atol=TOL, rtol=0)


def test_full_block_beats_partial_and_ignores_mask_mod(oracle_mod):
    """One key block listed both ways counts as full: mask_mod does not apply there."""
    B, H, S, D = 1, 1, 8, 4
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=5)
    one = np.ones((1, 1, 1), np.int32)
    blk = np.zeros((1, 1, 1, 1), np.int32)
    o_both, l_both = oracle_mod.fwd_block_sparse(q, k, v, one, blk, one, blk, mask_mod="causal", bm=8, bn=8)
    o_none, l_none = oracle_mod.fwd(q, k, v, mask_mod="none")
    np.testing.assert_allclose(o_both, o_none, atol=TOL, rtol=0)
    np.testing.assert_allclose(l_both, l_none, atol=TOL, rtol=0)
    o_part, l_part = oracle_mod.fwd_block_sparse(q, k, v, one, blk, None, None, mask_mod="causal", bm=8, bn=8)
    o_c, l_c = oracle_mod.fwd(q, k, v, mask_mod="causal")
    np.testing.assert_allclose(o_part, o_c, atol=TOL, rtol=0)
    np.testing.assert_allclose(l_part, l_c, atol=TOL, rtol=0)


@pytest.mark.parametrize("mask,window,offset", [("causal", 0, 0), ("sliding_window", 150, 0),
                                                ("kv_le_q_plus_offset", 0, -70), ("none", 0, 0)])
def test_every_block_partial_equals_mask_mod(oracle_mod, mask, window, offset):
    B, H, Sq, Skv, D = 1, 2, 300, 333, 8
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=9)
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    kn = np.full((1, 1, nq), nk, np.int32)
    ki = np.broadcast_to(np.arange(nk, dtype=np.int32)[::-1], (1, 1, nq, nk))
    o, lse = oracle_mod.fwd_block_sparse(q, k, v, kn, ki, mask_mod=mask, window=window, offset=offset)
    ro, rl = oracle_mod.fwd(q, k, v, mask_mod=mask, window=window, offset=offset)
    np.testing.assert_allclose(o, ro, atol=TOL, rtol=0)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(rl))
    fin = np.isfinite(rl)
    np.testing.assert_allclose(lse[fin], rl[fin], atol=TOL, rtol=0)


def test_every_block_full_equals_no_mask(oracle_mod):
    B, H, Sq, Skv, D = 2, 2, 140, 260, 8
    q, k, v = synth.qkv(B, H, 1, Sq, Skv, D, seed=10)
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    fn = np.full((1, 1, nq), nk, np.int32)
    fi = np.broadcast_to(np.arange(nk, dtype=np.int32), (1, 1, nq, nk))
    o, lse = oracle_mod.fwd_block_sparse(q, k, v, None, None, fn, fi, mask_mod="causal", score_mod="alibi")
    ro, rl = oracle_mod.fwd(q, k, v, mask_mod="none", score_mod="alibi")
    np.testing.assert_allclose(o, ro, atol=TOL, rtol=0)
    np.testing.assert_allclose(lse, rl, atol=TOL, rtol=0)


def test_empty_block_mask_gives_zero_rows(oracle_mod):
    B, H, Sq, Skv, D = 1, 2, 130, 129, 8
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=14)
    z = np.zeros((1, 1, 2), np.int32)
    zi = np.zeros((1, 1, 2, 2), np.int32)
    o, lse = oracle_mod.fwd_block_sparse(q, k, v, z, zi, z, zi)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("mask,window,offset", [("causal", 0, 0), ("sliding_window", 100, 0),
                                                ("kv_le_q_plus_offset", 0, 40)])
def test_tile_map_lists_equal_mask_mod(oracle_mod, mask, window, offset):
    """Dropping EMPTY tiles and not masking FULL ones changes nothing (the lists read
    off the analytic tile map reproduce the analytic mask)."""
    B, H, Sq, Skv, D = 1, 2, 385, 300, 8
    q, k, v = synth.qkv(B, H, 1, Sq, Skv, D, seed=15)
    tm = oracle_mod.tile_map(mask, Sq, Skv, window, offset)
    kn, ki, fn, fi = oracle_mod.block_mask_from_tile_map(tm, 1, 1)
    o, lse = oracle_mod.fwd_block_sparse(q, k, v, kn, ki, fn, fi, mask_mod=mask, window=window, offset=offset)
    ro, rl = oracle_mod.fwd(q, k, v, mask_mod=mask, window=window, offset=offset)
    np.testing.assert_allclose(o, ro, atol=TOL, rtol=0)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(rl))


def test_broadcast_lists_and_row_subset(oracle_mod):
    B, H, Sq, Skv, D, bm, bn = 2, 3, 20, 30, 8, 8, 8
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    rng = np.random.default_rng(3)
    kn, ki, fn, fi = _random_lists(rng, 1, 1, nq, nk, max_blocks=nk)
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=16)
    o1, l1 = oracle_mod.fwd_block_sparse(q, k, v, kn, ki, fn, fi, mask_mod="causal", bm=bm, bn=bn)
    tile = lambda a: np.tile(a, (B, H) + (1,) * (a.ndim - 2))
    o2, l2 = oracle_mod.fwd_block_sparse(q, k, v, tile(kn), tile(ki), tile(fn), tile(fi), mask_mod="causal",
                                         bm=bm, bn=bn)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    rows = [0, 7, 19, 20, B * H * Sq - 1]
    o3, l3 = oracle_mod.fwd_block_sparse(q, k, v, kn, ki, fn, fi, mask_mod="causal", bm=bm, bn=bn, rows=rows)
    np.testing.assert_array_equal(o3, o1.reshape(-1, D)[rows])
    np.testing.assert_array_equal(l3, l1.reshape(-1)[rows])
