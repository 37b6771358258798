"""Pins for the oracle's tensor-capturing mods.

FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod) on the generic flash-attention
kernel", Out of scope, names tensor-capturing mods as a later phase without defining any;
the two taken here are alibi with a captured per-head slope table, and a document mask
over packed sequences whose captured tensors are per-batch document boundaries.

Checked against things other than the oracle's own loops: a torch float64 softmax with
the bias / keep matrix the test builds independently (document ids by numpy searchsorted
on the boundaries), identities with already pinned mods (the built-in slopes; one
document covering everything == no mask / causal), and tile classes reduced from the
test's own keep matrix.
"""
import numpy as np
import pytest
import torch

import synth

TOL = 1e-12


def _torch_ref(q, k, v, scale, keep=None, slopes=None):
    B, H, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    kk = k.double().repeat_interleave(H // Hkv, dim=1)
    vv = v.double().repeat_interleave(H // Hkv, dim=1)
    s = torch.einsum("bhid,bhjd->bhij", q.double(), kk) * scale
    if slopes is not None:
        rel = torch.arange(Skv, dtype=torch.float64)[None, :] - torch.arange(Sq, dtype=torch.float64)[:, None]
        s = s + torch.as_tensor(slopes, dtype=torch.float64)[:, None, None] * rel
    if keep is None:
        keep = np.ones((B, H, Sq, Skv), bool)
    kt = torch.from_numpy(np.broadcast_to(keep, (B, H, Sq, Skv)).copy())
    s = s.masked_fill(~kt, float("-inf"))
    any_row = kt.any(-1)
    p = torch.softmax(s.masked_fill(~any_row[..., None], 0.0), -1) * any_row[..., None]
    return (p @ vv).numpy(), torch.logsumexp(s, -1).numpy(), any_row.numpy()


def _doc_ids(off, n):
    """Document of each position 0..n-1 under boundaries off (-1 outside every document)."""
    off = np.asarray(off)
    d = np.searchsorted(off, np.arange(n), side="right") - 1
    valid = (d >= 0) & (d < len(off) - 1)
    d = np.where(valid, d, -1)
    # a position at an empty document's boundary belongs to the next non-empty one
    for p in range(n):
        if d[p] >= 0 and not (off[d[p]] <= p < off[d[p] + 1]):
            d[p] = -1
    return d


def _doc_keep(off_q, off_kv, Sq, Skv, causal):
    dq, dk = _doc_ids(off_q, Sq), _doc_ids(off_kv, Skv)
    keep = (dq[:, None] == dk[None, :]) & (dq[:, None] >= 0)
    if causal:
        keep &= np.arange(Skv)[None, :] <= np.arange(Sq)[:, None]
    return keep


def _check(o, lse, ro, rl, live):
    np.testing.assert_allclose(o, ro, atol=TOL, rtol=0)
    assert np.all(np.isneginf(lse[~live])) and np.all(o[~live] == 0.0)
    np.testing.assert_allclose(lse[live], rl[live], atol=TOL, rtol=0)


def test_slope_table_equal_to_builtin_is_alibi(oracle_mod):
    B, H, S, D = 1, 8, 19, 8
    q, k, v = synth.qkv(B, H, 2, S, S, D, seed=31)
    table = [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]
    o1, l1 = oracle_mod.fwd(q, k, v, scale=0.3, score_mod="alibi", mask_mod="causal", alibi_slopes=table)
    o2, l2 = oracle_mod.fwd(q, k, v, scale=0.3, score_mod="alibi", mask_mod="causal")
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_random_slope_table_equals_torch(oracle_mod):
    B, H, Sq, Skv, D = 2, 4, 13, 21, 8
    q, k, v = synth.qkv(B, H, 4, Sq, Skv, D, seed=32)
    table = np.array([0.7, -0.25, 0.0, 1.5])
    o, lse = oracle_mod.fwd(q, k, v, scale=0.4, score_mod="alibi", alibi_slopes=table)
    ro, rl, live = _torch_ref(q, k, v, 0.4, slopes=table)
    _check(o, lse, ro, rl, live)


def test_zero_slopes_equal_no_mod(oracle_mod):
    q, k, v = synth.qkv(1, 3, 3, 9, 11, 8, seed=33)
    o1, l1 = oracle_mod.fwd(q, k, v, scale=0.5, score_mod="alibi", alibi_slopes=[0.0, 0.0, 0.0])
    o2, l2 = oracle_mod.fwd(q, k, v, scale=0.5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


OFFS = {
    # per batch row: boundaries of the query positions (and of the keys, same unless given)
    "packed": ([[0, 5, 6, 17, 30], [0, 12, 12, 25, 30]], None),          # an empty document
    "tail_unassigned": ([[0, 9, 20, 24, 24], [0, 3, 4, 10, 22]], None),   # positions >= last end
    "cross": ([[0, 4, 10, 15, 30], [0, 10, 11, 20, 30]], [[0, 9, 9, 20, 37], [0, 2, 30, 31, 37]]),
}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", list(OFFS))
def test_document_masks_equal_torch(oracle_mod, case, causal):
    off_q, off_kv = OFFS[case]
    B, H, D = 2, 2, 8
    Sq = 30
    Skv = 37 if case == "cross" else 30
    q, k, v = synth.qkv(B, H, 1, Sq, Skv, D, seed=34)
    mask = "document_causal" if causal else "document"
    o, lse = oracle_mod.fwd(q, k, v, scale=0.45, mask_mod=mask, score_mod="alibi", doc_offsets=off_q,
                            doc_offsets_kv=off_kv)
    keep = np.stack([_doc_keep(off_q[b], (off_kv or off_q)[b], Sq, Skv, causal) for b in range(B)])[:, None]
    ro, rl, live = _torch_ref(q, k, v, 0.45, keep=keep, slopes=[2.0 ** (-4.0 * (h + 1)) for h in range(H)])
    _check(o, lse, ro, rl, live)
    assert (~live).any() or case == "packed"


def test_one_document_equals_plain_masks(oracle_mod):
    B, H, S, D = 2, 2, 40, 8
    q, k, v = synth.qkv(B, H, 2, S, S, D, seed=35)
    off = [[0, S], [0, S]]
    for doc_mask, plain in (("document", "none"), ("document_causal", "causal")):
        o1, l1 = oracle_mod.fwd(q, k, v, scale=0.2, mask_mod=doc_mask, doc_offsets=off)
        o2, l2 = oracle_mod.fwd(q, k, v, scale=0.2, mask_mod=plain)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_document_mask_matrix_and_tile_map(oracle_mod, causal):
    off_q, off_kv = [0, 100, 100, 290, 300], [0, 130, 131, 333, 400]
    Sq, Skv = 300, 400
    mask = "document_causal" if causal else "document"
    keep = _doc_keep(off_q, off_kv, Sq, Skv, causal)
    got = oracle_mod.mask_matrix(mask, Sq, Skv, doc_offsets=off_q, doc_offsets_kv=off_kv)
    np.testing.assert_array_equal(got.astype(bool), keep)
    bm = bn = 64
    tm = oracle_mod.tile_map(mask, Sq, Skv, bm=bm, bn=bn, doc_offsets=off_q, doc_offsets_kv=off_kv)
    for t in range(tm.shape[0]):
        for u in range(tm.shape[1]):
            blk = np.zeros((bm, bn), bool)
            sub = keep[t * bm:(t + 1) * bm, u * bn:(u + 1) * bn]
            blk[:sub.shape[0], :sub.shape[1]] = sub
            rows = min(bm, Sq - t * bm)
            want = 0 if not blk.any() else (1 if blk[:rows].all() else 2)
            assert tm[t, u] == want, (t, u)


def test_document_block_sparse_uses_captured_rule(oracle_mod):
    """Partial blocks of a block mask apply the captured document rule."""
    B, H, S, D = 1, 2, 300, 8
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=36)
    off = [[0, 70, 200, 300]]
    nq = nk = 3
    kn = np.full((1, 1, nq), nk, np.int32)
    ki = np.broadcast_to(np.arange(nk, dtype=np.int32), (1, 1, nq, nk)).copy()
    o1, l1 = oracle_mod.fwd_block_sparse(q, k, v, kn, ki, mask_mod="document_causal", doc_offsets=off)
    o2, l2 = oracle_mod.fwd(q, k, v, mask_mod="document_causal", doc_offsets=off)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
