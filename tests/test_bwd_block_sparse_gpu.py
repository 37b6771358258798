"""GPU parity of flex_attn_bwd_block_sparse (the backward of the BlockMask forward)
against the fp64 oracle (oracle.bwd_block_sparse), through the C ABI.

Block sparsity and the backward are both named as later phases on FlyDSL PR 931 "Add
flex_attention (score_mod / mask_mod) on the generic flash-attention kernel" (Out of
scope).  The kernels take O and LSE from flex_attn_fwd_block_sparse, as a caller would.
Tolerances as in test_bwd_gpu.py.  Besides random lists (duplicates, indices naming no
block, over-long and negative counts) the tests check identities with the dense
backward that must hold bit for bit: lists read off the analytic tile map, and every
block full under a mask_mod, visit the same tiles in the same order as flex_attn_bwd.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.helpers import random_block_lists
from tests.test_bwd_gpu import _check

pytestmark = pytest.mark.gpu


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _dev(*arrays):
    return [None if a is None else torch.as_tensor(np.ascontiguousarray(a)).cuda() for a in arrays]


def _run(q, k, v, dout, lists, scale, **mods):
    fa = _fa()
    m = dict(mods)
    for key in ("alibi_slopes", "doc_offsets"):
        if m.get(key) is not None:
            m[key] = torch.as_tensor(m[key]).cuda()
    qd, kd, vd, od = (t.cuda() for t in (q, k, v, dout))
    L = _dev(*lists)
    o, lse = fa.fwd_block_sparse(qd, kd, vd, *L, scale=scale, **m)
    dq, dk, dv = fa.bwd_block_sparse(qd, kd, vd, o, lse, od, *L, scale=scale, **m)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return dq, dk, dv


MODS = [dict(mask_mod="none"), dict(mask_mod="causal"), dict(mask_mod="causal", score_mod="alibi"),
        dict(mask_mod="sliding_window", window=150), dict(mask_mod="kv_le_q_plus_offset", offset=-60),
        dict(score_mod="alibi", alibi_slopes=np.array([0.25, -0.0625, 0.5, 0.0], np.float32)),
        dict(mask_mod="document_causal", doc_offsets=np.array([[0, 90, 90, 250, 300], [0, 1, 200, 201, 300]],
                                                                np.int32))]


@pytest.mark.parametrize("mods", MODS, ids=lambda m: "-".join(f"{k}={v}" for k, v in m.items()
                                                              if k in ("mask_mod", "score_mod")) +
                         ("-slopes" if "alibi_slopes" in m else ""))
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f16")])
def test_random_lists(mods, D, dtype):
    """Sq = 300, Skv = 700 (three query tiles, six key tiles, ragged), GQA 4/2."""
    B, H, Hkv, Sq, Skv = 2, 4, 2, 300, 700
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    rng = np.random.default_rng(700 + D + len(mods))
    lists = random_block_lists(rng, B, H, nq, nk, max_blocks=nk + 2, p_full=0.35, p_part=0.35)
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=91, dtype=dtype)
    dout = synth.normal_tensor((B, H, Sq, D), 92, dtype=dtype)
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = _run(q, k, v, dout, lists, scale, **mods)
    rq, rk, rv = oracle.bwd_block_sparse(q, k, v, dout, *lists, scale=scale, **mods)
    _check("dq", dq, rq), _check("dk", dk, rk), _check("dv", dv, rv)


@pytest.mark.parametrize("mask,window,offset", [("causal", 0, 0), ("sliding_window", 300, 0),
                                                ("kv_le_q_plus_offset", 0, -100), ("none", 0, 0)])
def test_tile_map_lists_match_dense_backward_bitwise(mask, window, offset):
    """Lists read off the analytic tile map: the same tiles, classes and order as the
    dense backward, so the gradients agree bit for bit."""
    fa = _fa()
    B, H, Hkv, S, D = 1, 4, 2, 640, 128
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=93, device="cuda")
    dout = synth.normal_tensor((B, H, S, D), 94, dtype="bf16", device="cuda")
    tm = oracle.tile_map(mask, S, S, window=window, offset=offset)
    L = _dev(*oracle.block_mask_from_tile_map(tm, 1, 1))
    mods = dict(mask_mod=mask, window=window, offset=offset)
    o, lse = fa.fwd(q, k, v, **mods)
    ref = fa.bwd(q, k, v, o, lse, dout, **mods)
    got = fa.bwd_block_sparse(q, k, v, o, lse, dout, *L, **mods)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_all_full_lists_ignore_mask_mod_bitwise():
    """Every block full under mask_mod=causal == the unmasked backward (Skv ragged)."""
    fa = _fa()
    B, H, Sq, Skv, D = 1, 2, 300, 1000, 64
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=95, device="cuda")
    dout = synth.normal_tensor((B, H, Sq, D), 96, dtype="bf16", device="cuda")
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    fn = torch.full((1, 1, nq), nk, dtype=torch.int32, device="cuda")
    fi = torch.arange(nk, dtype=torch.int32, device="cuda").expand(1, 1, nq, nk).contiguous()
    o, lse = fa.fwd(q, k, v)
    ref = fa.bwd(q, k, v, o, lse, dout)
    got = fa.bwd_block_sparse(q, k, v, o, lse, dout, None, None, fn, fi, mask_mod="causal")
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_empty_lists_give_zero_gradients():
    fa = _fa()
    B, H, S, D = 1, 2, 200, 128
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=97, device="cuda")
    dout = synth.normal_tensor((B, H, S, D), 98, dtype="bf16", device="cuda")
    z = torch.zeros((1, 1, 2), dtype=torch.int32, device="cuda")
    zi = torch.zeros((1, 1, 2, 1), dtype=torch.int32, device="cuda")
    o, lse = fa.fwd_block_sparse(q, k, v, z, zi, z, zi)
    dq, dk, dv = fa.bwd_block_sparse(q, k, v, o, lse, dout, z, zi, z, zi)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    for g in (dq, dk, dv):
        assert torch.all(g == 0)


def test_long_8192_random_lists_sampled_groups():
    """B2 H32 S8192 D128 with random per-head lists (about half of the key blocks of each
    query tile, a third of them partial under causal): two whole (b, head) groups."""
    fa = _fa()
    B, H, S, D = 2, 32, 8192, 128
    nq = S // 128
    rng = np.random.default_rng(4104)
    sel = rng.random((B, H, nq, nq)) < 0.5
    part = sel & (rng.random((B, H, nq, nq)) < 0.33)
    full = sel & ~part

    def lists(m):
        return m.sum(-1).astype(np.int32), np.argsort(~m, axis=-1, kind="stable").astype(np.int32)
    L = [*lists(part), *lists(full)]
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=4000, sigma=0.5, device="cuda")
    dout = synth.normal_tensor((B, H, S, D), 4103, dtype="bf16", device="cuda")
    scale = 1.0 / math.sqrt(D)
    Ld = _dev(*L)
    o, lse = fa.fwd_block_sparse(q, k, v, *Ld, scale=scale, mask_mod="causal")
    dq, dk, dv = fa.bwd_block_sparse(q, k, v, o, lse, dout, *Ld, scale=scale, mask_mod="causal")
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    groups = [(0, 5), (1, 30)]
    rq, rk, rv = oracle.bwd_block_sparse(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), *L, scale=scale,
                                         mask_mod="causal", groups=groups)
    dq = torch.stack([dq[b, hk:hk + 1] for b, hk in groups])
    dk = torch.stack([dk[b, hk] for b, hk in groups])
    dv = torch.stack([dv[b, hk] for b, hk in groups])
    _check("dq", dq, rq), _check("dk", dk, rk), _check("dv", dv, rv)
