"""Pins for the oracle's block-sparse backward (the gradients of the BlockMask forward).

FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod) on the generic flash-attention
kernel", "Out of scope (future phases)", names both block sparsity and the backward pass
as later phases; the oracle composes its two readings: the backward of the forward whose
keep rule is PyTorch's BlockMask convention.  Checked against:
  * torch float64 autograd through a softmax whose keep matrix the test builds block by
    block from Python sets of the listed indices (random lists with duplicates, indices
    naming no block, over-long and negative counts; every mask_mod; alibi; GQA; bf16/f16),
  * reductions to the pinned dense backward: every block full == no mask, every block
    partial == mask_mod, lists read off the analytic tile map == mask_mod,
  * the empty mask: every gradient exactly zero.
"""
import numpy as np
import pytest
import torch

import synth
from tests.helpers import random_block_lists as _random_lists
from tests.test_oracle_block_pins import _dense_keep
from tests.test_oracle_bwd_pins import _autograd, _slopes

TOL = 1e-12


@pytest.mark.parametrize("mask,window,offset,score", [
    ("none", 0, 0, "none"), ("causal", 0, 0, "alibi"), ("sliding_window", 6, 0, "none"),
    ("kv_le_q_plus_offset", 0, -5, "alibi")])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_block_bwd_equals_autograd(oracle_mod, mask, window, offset, score, dtype):
    B, H, Hkv, Sq, Skv, D, bm, bn = 2, 4, 2, 23, 37, 8, 4, 8
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    rng = np.random.default_rng(4321 + len(mask) + offset)
    kn, ki, fn, fi = _random_lists(rng, B, H, nq, nk, max_blocks=nk + 1)
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=78, dtype=dtype)
    dout = synth.normal_tensor((B, H, Sq, D), 79, dtype="bf16" if dtype == torch.bfloat16 else "f16")
    dq, dk, dv = oracle_mod.bwd_block_sparse(q, k, v, dout, kn, ki, fn, fi, scale=0.37, score_mod=score,
                                             mask_mod=mask, window=window, offset=offset, bm=bm, bn=bn)
    elem = oracle_mod.mask_matrix(mask, Sq, Skv, window, offset).astype(bool)
    keep = _dense_keep(elem, kn, ki, fn, fi, B, H, Sq, Skv, bm, bn)
    assert keep.any() and not keep.all()
    rq, rk, rv = _autograd(q, k, v, dout, 0.37, keep=keep, slopes=_slopes(H) if score == "alibi" else None)
    np.testing.assert_allclose(dq, rq, atol=TOL, rtol=0)
    np.testing.assert_allclose(dk, rk, atol=TOL, rtol=0)
    np.testing.assert_allclose(dv, rv, atol=TOL, rtol=0)


def _grads_equal(a, b):
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, atol=TOL, rtol=0)


def test_block_bwd_reduces_to_dense(oracle_mod):
    B, H, Hkv, Sq, Skv, D = 1, 2, 1, 300, 333, 8
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=80)
    dout = synth.normal_tensor((B, H, Sq, D), 81, dtype="bf16")
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    every = np.broadcast_to(np.arange(nk, dtype=np.int32)[::-1], (1, 1, nq, nk))
    count = np.full((1, 1, nq), nk, np.int32)
    # every block full == no mask (mask_mod ignored on full blocks)
    _grads_equal(oracle_mod.bwd_block_sparse(q, k, v, dout, None, None, count, every, mask_mod="causal",
                                             score_mod="alibi"),
                 oracle_mod.bwd(q, k, v, dout, mask_mod="none", score_mod="alibi"))
    # every block partial == mask_mod
    for mask, window, offset in (("causal", 0, 0), ("sliding_window", 150, 0), ("kv_le_q_plus_offset", 0, -70)):
        _grads_equal(oracle_mod.bwd_block_sparse(q, k, v, dout, count, every, mask_mod=mask, window=window,
                                                 offset=offset),
                     oracle_mod.bwd(q, k, v, dout, mask_mod=mask, window=window, offset=offset))
        # lists read off the analytic tile map (EMPTY tiles dropped, FULL ones unmasked)
        tm = oracle_mod.tile_map(mask, Sq, Skv, window, offset)
        lists = oracle_mod.block_mask_from_tile_map(tm, 1, 1)
        _grads_equal(oracle_mod.bwd_block_sparse(q, k, v, dout, *lists, mask_mod=mask, window=window,
                                                 offset=offset),
                     oracle_mod.bwd(q, k, v, dout, mask_mod=mask, window=window, offset=offset))


def test_block_bwd_empty_mask_and_groups(oracle_mod):
    B, H, Hkv, Sq, Skv, D, bm, bn = 2, 4, 2, 20, 30, 8, 8, 8
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=82)
    dout = synth.normal_tensor((B, H, Sq, D), 83, dtype="bf16")
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    z, zi = np.zeros((1, 1, nq), np.int32), np.zeros((1, 1, nq, 2), np.int32)
    for g in oracle_mod.bwd_block_sparse(q, k, v, dout, z, zi, z, zi, bm=bm, bn=bn):
        assert np.all(g == 0.0)
    rng = np.random.default_rng(5)
    lists = _random_lists(rng, B, H, nq, nk, max_blocks=nk)
    dq, dk, dv = oracle_mod.bwd_block_sparse(q, k, v, dout, *lists, mask_mod="causal", bm=bm, bn=bn)
    gq, gk, gv = oracle_mod.bwd_block_sparse(q, k, v, dout, *lists, mask_mod="causal", bm=bm, bn=bn,
                                             groups=[(1, 0), (0, 1)])
    G = H // Hkv
    np.testing.assert_array_equal(gq[0], dq[1, 0:G])
    np.testing.assert_array_equal(gq[1], dq[0, G:2 * G])
    np.testing.assert_array_equal(gk[0], dk[1, 0])
    np.testing.assert_array_equal(gv[1], dv[0, 1])
