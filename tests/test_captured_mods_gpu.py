"""GPU parity of the tensor-capturing mods against the fp64 oracle.

Tensor-capturing mods are named as a later phase on FlyDSL PR 931 "Add flex_attention
(score_mod / mask_mod) on the generic flash-attention kernel" (Out of scope). The two
built: alibi with a captured per-head slope tensor, and document masks over packed
sequences whose captured tensors are per-batch document boundaries (optionally causal).

Covers: random slope tables (negative, zero); packed documents with empty documents,
one-token documents, unassigned tail positions and boundaries off the 128 grid; separate
key boundaries (cross attention); D 64/128, bf16/f16, GQA; one all-covering document is
bit-identical to the plain kernels; kernel tile maps and element masks equal the
oracle's bit for bit; block lists read off the document tile map give the document
kernel's bits; S=8192 packed documents on sampled rows; boundaries that break the
non-decreasing precondition run cleanly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.helpers import compare, gather_rows, sample_rows

pytestmark = pytest.mark.gpu


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _run(q, k, v, scale, blocks=None, **mods):
    fa = _fa()
    dev = torch.device("cuda")
    m = dict(mods)
    for key in ("alibi_slopes", "doc_offsets", "doc_offsets_kv"):
        if m.get(key) is not None:
            m[key] = torch.as_tensor(m[key]).to(dev)
    if blocks is None:
        o, lse = fa.fwd(q.to(dev), k.to(dev), v.to(dev), scale=scale, **m)
    else:
        lists = [None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in blocks]
        o, lse = fa.fwd_block_sparse(q.to(dev), k.to(dev), v.to(dev), *lists, scale=scale, **m)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return o, lse


def _packed(rng, B, S, n_docs, lo=1, hi=None):
    """int32 [B, n_docs + 1] boundaries: sorted cut points (repeats = empty documents)."""
    out = np.zeros((B, n_docs + 1), np.int32)
    for b in range(B):
        cuts = np.sort(rng.integers(lo, (hi or S), n_docs - 1))
        out[b, 1:-1] = cuts
        out[b, -1] = S
    return out


SLOPES = np.array([0.5, -0.25, 0.0, 1.0 / 64, 2.0, -1.0 / 32, 0.125, 0.03125], np.float32)


@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("sliding_window", 150)])
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f16")])
def test_slope_table(mask, window, D, dtype):
    B, H, Hkv, Sq, Skv = 2, 8, 2, 300, 700
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=synth.case_seed(50, D), dtype=dtype)
    mods = dict(score_mod="alibi", mask_mod=mask, window=window, alibi_slopes=SLOPES)
    o, lse = _run(q, k, v, 1.0 / math.sqrt(D), **mods)
    ro, rl = oracle.fwd(q, k, v, scale=1.0 / math.sqrt(D), **mods)
    compare(o, lse, ro, rl, f"slopes {mask}")


def _doc_cases():
    rng = np.random.default_rng(51)
    return {
        "packed": (_packed(rng, 2, 700, 6), None, 700, 700),
        "empty_and_tiny": (np.array([[0, 1, 1, 130, 131, 500, 700], [0, 0, 256, 256, 257, 699, 700]], np.int32),
                           None, 700, 700),
        "tail_unassigned": (np.array([[0, 200, 450, 451, 600], [0, 10, 300, 301, 333]], np.int32), None, 700, 700),
        "cross": (np.array([[0, 100, 260, 300, 300], [0, 50, 51, 200, 300]], np.int32),
                  np.array([[0, 400, 410, 800, 1000], [0, 1, 700, 900, 1000]], np.int32), 300, 1000),
    }


DOCS = _doc_cases()


@pytest.mark.parametrize("case", list(DOCS))
@pytest.mark.parametrize("mask", ["document", "document_causal"])
@pytest.mark.parametrize("D,dtype,score", [(128, "bf16", "none"), (64, "f16", "alibi"), (128, "f16", "alibi")])
def test_document_masks(case, mask, D, dtype, score):
    off_q, off_kv, Sq, Skv = DOCS[case]
    B, H, Hkv = 2, 4, 2
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=synth.case_seed(52, D), dtype=dtype)
    mods = dict(score_mod=score, mask_mod=mask, doc_offsets=off_q, doc_offsets_kv=off_kv)
    o, lse = _run(q, k, v, 1.0 / math.sqrt(D), **mods)
    ro, rl = oracle.fwd(q, k, v, scale=1.0 / math.sqrt(D), **mods)
    compare(o, lse, ro, rl, f"{case} {mask}")


@pytest.mark.parametrize("doc_mask,plain", [("document", "none"), ("document_causal", "causal")])
def test_one_document_bit_exact_with_plain_mask(doc_mask, plain):
    fa = _fa()
    B, H, S, D = 2, 4, 1000, 128
    q, k, v = synth.qkv(B, H, 2, S, S, D, seed=53, device="cuda")
    off = torch.tensor([[0, S], [0, S]], dtype=torch.int32, device="cuda")
    o1, l1 = fa.fwd(q, k, v, scale=0.1, score_mod="alibi", mask_mod=doc_mask, doc_offsets=off)
    o2, l2 = fa.fwd(q, k, v, scale=0.1, score_mod="alibi", mask_mod=plain)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("case", ["packed", "empty_and_tiny", "cross"])
@pytest.mark.parametrize("mask", ["document", "document_causal"])
def test_tile_map_and_mask_eval_bit_exact(case, mask):
    fa = _fa()
    off_q, off_kv, Sq, Skv = DOCS[case]
    oq, okv = off_q[:1], None if off_kv is None else off_kv[:1]
    want_keep = oracle.mask_matrix(mask, Sq, Skv, doc_offsets=oq[0], doc_offsets_kv=None if okv is None else okv[0])
    dq = torch.from_numpy(oq).cuda()
    dkv = None if okv is None else torch.from_numpy(okv).cuda()
    keep = fa.mask_eval(mask, Sq, Skv, doc_offsets=dq, doc_offsets_kv=dkv)
    np.testing.assert_array_equal(keep.cpu().numpy(), want_keep)
    want_map = oracle.tile_map(mask, Sq, Skv, doc_offsets=oq[0], doc_offsets_kv=None if okv is None else okv[0])
    q, k, v = synth.qkv(1, 2, 2, Sq, Skv, 64, seed=54, device="cuda")
    tmap = torch.full((want_map.size,), 77, dtype=torch.uint8, device="cuda")
    fa.fwd(q, k, v, mask_mod=mask, doc_offsets=dq, doc_offsets_kv=dkv, tile_map=tmap)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(tmap.cpu().numpy().reshape(want_map.shape), want_map)


def test_block_lists_from_document_tile_map_bit_exact():
    fa = _fa()
    off_q, _, S, _ = DOCS["packed"]
    B, H, D = 2, 4, 128
    q, k, v = synth.qkv(B, H, 2, S, S, D, seed=55, device="cuda")
    # one list per batch row (documents differ per batch), shared by the heads
    lists = [oracle.block_mask_from_tile_map(oracle.tile_map("document_causal", S, S, doc_offsets=off_q[b]), 1, 1)
             for b in range(B)]
    kn, ki, fn, fi = (np.concatenate([l[i] for l in lists], axis=0) for i in range(4))
    mods = dict(score_mod="alibi", mask_mod="document_causal", doc_offsets=off_q)
    o_b, l_b = _run(q, k, v, 0.1, blocks=(kn, ki, fn, fi), **mods)
    o_a, l_a = _run(q, k, v, 0.1, **mods)
    assert torch.equal(o_b, o_a) and torch.equal(l_b, l_a)


@pytest.mark.parametrize("mask", ["document", "document_causal"])
def test_long_8192_packed_sampled(mask):
    B, H, S, D = 2, 32, 8192, 128
    rng = np.random.default_rng(56)
    off = _packed(rng, B, S, 9)
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=synth.case_seed(56, 1), device="cuda")
    scale = 1.0 / math.sqrt(D)
    o, lse = _run(q, k, v, scale, score_mod="alibi", mask_mod=mask, doc_offsets=off)
    must = [(0, 0, int(off[0, 1]) - 1), (0, 0, int(off[0, 1])), (1, 31, S - 1), (1, 3, int(off[1, 4]))]
    rows = sample_rows(B, H, S, 192, seed=57, must=must)
    ro, rl = oracle.fwd(q.cpu(), k.cpu(), v.cpu(), scale=scale, score_mod="alibi", mask_mod=mask,
                        doc_offsets=off, rows=rows)
    compare(gather_rows(o, rows), gather_rows(lse, rows), ro, rl, mask)


def test_unsorted_boundaries_run_cleanly():
    """Boundaries that break the non-decreasing precondition: the keys kept are
    unspecified, but the kernel reads only the boundaries given and ends normally."""
    B, H, S, D = 1, 2, 500, 64
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=58)
    off = np.array([[0, 300, 100, 450, 200, 500]], np.int32)
    o, lse = _run(q, k, v, 0.125, mask_mod="document_causal", doc_offsets=off)
    assert not torch.isnan(o.float()).any() and not torch.isnan(lse).any()
