"""GPU parity of flex_attn_fwd_fp8 (e4m3 Q/K/V, per-tensor descales, bf16 O).

FP8 flex paths are named as a later phase on FlyDSL PR 931 "Add flex_attention (score_mod
/ mask_mod) on the generic flash-attention kernel" (Out of scope). The oracle computes the
exact definition on the dequantized inputs (P unrounded); the kernel rounds P to e4m3 for
the P.V product. Tolerance per element, derived from that rounding: P' = P * 2^(6..8)
keeps a relative error of 2^-4 for normal e4m3 values and an absolute error of 2^-10 in
P' (2^-16 in P) below them, so
    |O - O_ref| <= descale_v * (2^-4 * (P |v8|) + 2^-16 * (keep |v8|)) * 1.05
                   + 2^-8 |O_ref| + 1e-4            (bf16 output rounding, fp32 sums),
checked element by element with the oracle's P; LSE (unaffected by the rounding of P)
within 1e-2; rows without keys O = +0 and LSE = -inf exactly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _inputs(B, H, Hkv, Sq, Skv, seed, spread=1.0, sigma=1.0, device="cpu", D=128):
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=seed, sigma=sigma, device=device)
    return tuple((t.float() * spread).to(torch.float8_e4m3fn).cpu() for t in (q, k, v))


def _check(q8, k8, v8, o, lse, dq, dk, dv, scale, rows=None, **mods):
    ro, rl = oracle.fwd_fp8(q8, k8, v8, descale_q=dq, descale_k=dk, descale_v=dv, scale=scale, rows=rows, **mods)
    # the oracle's probabilities on the same values (every e4m3 value is exact in bf16)
    bf = lambda t: t.to(torch.bfloat16)
    _, _, P = oracle.fwd(bf(q8), bf(k8), bf(v8), scale=scale * dq * dk, rows=rows, want_probs=True, **mods)
    B, H, Sq, D = q8.shape
    G = H // k8.shape[1]
    av = np.abs(v8.double().numpy())  # [B, Hkv, Skv, D]
    if rows is None:
        av_rows = np.repeat(av, G, axis=1)                      # [B, H, Skv, D]
        Pm = P.reshape(B, H, Sq, -1)
        bound = dv * (2.0 ** -4 * np.einsum("bhij,bhjd->bhid", Pm, av_rows)
                      + 2.0 ** -16 * np.einsum("bhij,bhjd->bhid", (Pm > 0).astype(np.float64), av_rows))
        got = o.float().cpu().numpy().astype(np.float64)
        lg = lse.cpu().numpy().astype(np.float64)
    else:
        rows = np.asarray(rows)
        b_idx = rows // (H * Sq)
        hk_idx = ((rows // Sq) % H) // G
        bound = np.zeros((rows.size, D))
        for b in np.unique(b_idx):                              # one product per (batch, kv head)
            for hk in np.unique(hk_idx[b_idx == b]):
                sel = (b_idx == b) & (hk_idx == hk)
                Pg = P[sel]
                bound[sel] = dv * (2.0 ** -4 * (Pg @ av[b, hk]) + 2.0 ** -16 * ((Pg > 0).astype(np.float64) @ av[b, hk]))
        got = o.reshape(-1, D)[torch.as_tensor(rows, device=o.device)].float().cpu().numpy().astype(np.float64)
        lg = lse.reshape(-1)[torch.as_tensor(rows, device=lse.device)].cpu().numpy().astype(np.float64)
        ro, rl = ro.reshape(got.shape), rl.reshape(lg.shape)
    tol = 1.05 * bound + 2.0 ** -8 * np.abs(ro) + 1e-4
    err = np.abs(got - ro)
    assert not np.isnan(got).any()
    worst = float((err / tol).max())
    assert worst <= 1.0, f"O error exceeds the e4m3 bound (worst ratio {worst:.3f})"
    dead = np.isneginf(rl)
    assert np.array_equal(np.isneginf(lg), dead)
    assert np.all(got[dead] == 0.0)
    if (~dead).any():
        assert float(np.abs(lg[~dead] - rl[~dead]).max()) <= 1e-2
    return float(err.mean())


MODS = [dict(), dict(mask_mod="causal"), dict(mask_mod="causal", score_mod="alibi"),
        dict(mask_mod="sliding_window", window=150), dict(mask_mod="kv_le_q_plus_offset", offset=-60),
        dict(score_mod="alibi", alibi_slopes=np.array([0.25, -0.125, 0.0625, 0.5], np.float32))]


@pytest.mark.parametrize("mods", MODS, ids=lambda m: "-".join(f"{k}" for k in m) or "no_mod")
@pytest.mark.parametrize("desc", [(1.0, 1.0, 1.0), (0.5, 2.0, 0.25), (0.37, 1.3, 0.71)])
def test_ragged_gqa(mods, desc):
    fa = _fa()
    B, H, Hkv, Sq, Skv = 2, 4, 2, 300, 700
    q8, k8, v8 = _inputs(B, H, Hkv, Sq, Skv, seed=97)
    dq, dk, dv = desc
    scale = 1.0 / math.sqrt(128)
    m = dict(mods)
    if m.get("alibi_slopes") is not None:
        m["alibi_slopes"] = torch.from_numpy(m["alibi_slopes"]).cuda()
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), descale_q=dq, descale_k=dk, descale_v=dv, scale=scale, **m)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    _check(q8, k8, v8, o, lse, dq, dk, dv, scale, **mods)


@pytest.mark.parametrize("mods", MODS[:5], ids=lambda m: "-".join(f"{k}" for k in m) or "no_mod")
def test_ragged_gqa_d64(mods):
    """Head dim 64: the tiles stay 128 bytes wide and TMA pads Q, K and V^T with zeros."""
    fa = _fa()
    B, H, Hkv, Sq, Skv = 2, 4, 2, 300, 700
    q8, k8, v8 = _inputs(B, H, Hkv, Sq, Skv, seed=96, D=64)
    scale = 0.125
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), descale_q=0.5, descale_k=2.0, descale_v=0.75, scale=scale,
                        **mods)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    assert tuple(o.shape) == (B, H, Sq, 64)
    _check(q8, k8, v8, o, lse, 0.5, 2.0, 0.75, scale, **mods)


def test_d64_2048_sampled():
    fa = _fa()
    B, H, S = 2, 32, 2048
    q8, k8, v8 = _inputs(B, H, 8, S, S, seed=104, device="cuda", D=64)
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), mask_mod="causal")
    torch.cuda.synchronize()
    rows = _sampled_rows(B, H, S, 2048, 105, [(0, 0, 0), (0, 0, 127), (0, 0, 128), (1, 31, 2047)])
    _check(q8, k8, v8, o, lse, 1.0, 1.0, 1.0, 0.125, rows=rows, mask_mod="causal")


def test_rows_without_keys():
    fa = _fa()
    q8, k8, v8 = _inputs(1, 2, 2, 250, 1024, seed=98)
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), scale=0.1, mask_mod="kv_le_q_plus_offset", offset=-300)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_peaked_scores_wide_range():
    """Larger scores (values spread x4): P concentrates on few keys, where the 8-bit
    rounding of P matters most."""
    fa = _fa()
    q8, k8, v8 = _inputs(1, 4, 4, 256, 512, seed=99, spread=4.0)
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), scale=0.125, mask_mod="causal")
    torch.cuda.synchronize()
    _check(q8, k8, v8, o, lse, 1.0, 1.0, 1.0, 0.125, mask_mod="causal")


def _sampled_rows(B, H, S, n, seed, fixed):
    """n seeded random rows plus the fixed (b, h, i) rows, as flat indices."""
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(B * H * S, n, replace=False).tolist())
    pick.update((b * H + h) * S + i for b, h, i in fixed if i < S)
    return np.array(sorted(pick), dtype=np.int64)


@pytest.mark.parametrize("mods", [dict(mask_mod="causal"), dict()], ids=["causal", "no_mod"])
def test_mha_2048_sampled(mods):
    """B2 H32 S2048: 2048 seeded rows plus the first and last rows of the first and last
    query-tile pairs."""
    fa = _fa()
    B, H, S = 2, 32, 2048
    q8, k8, v8 = _inputs(B, H, H, S, S, seed=100, device="cuda")
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), descale_q=0.5, descale_k=0.5, descale_v=2.0, **mods)
    torch.cuda.synchronize()
    fixed = [(0, 0, 0), (0, 0, 127), (0, 0, 128), (0, 0, 255), (0, 0, 256), (1, 31, 1792), (1, 31, 2047),
             (1, 7, 1023), (1, 7, 1024)]
    rows = _sampled_rows(B, H, S, 2048, 101, fixed)
    _check(q8, k8, v8, o, lse, 0.5, 0.5, 2.0, 1.0 / math.sqrt(128), rows=rows, **mods)


@pytest.mark.parametrize("mods", [dict(), dict(mask_mod="causal"), dict(score_mod="alibi"),
                                  dict(mask_mod="sliding_window", window=1024)],
                         ids=["no_mod", "causal", "alibi", "window1024"])
def test_long_8192_sampled(mods):
    """The long-context shape (B2 H32 S8192, N(0, 0.5^2) rounded to e4m3) on 2048 seeded
    rows plus rows 0, 127, 128, 8191, the window edges and the first/last tile pairs."""
    fa = _fa()
    B, H, S = 2, 32, 8192
    q8, k8, v8 = _inputs(B, H, H, S, S, seed=102, sigma=0.5, device="cuda")
    scale = 1.0 / math.sqrt(128)
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), scale=scale, **mods)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    fixed = [(0, 0, 0), (0, 0, 127), (0, 0, 128), (0, 0, 255), (0, 0, 256), (1, 31, 8191), (1, 31, 7936),
             (0, 17, 1023), (0, 17, 1024), (0, 17, 1025), (1, 2, 4095)]
    rows = _sampled_rows(B, H, S, 2048, 103, fixed)
    _check(q8, k8, v8, o, lse, 1.0, 1.0, 1.0, scale, rows=rows, **mods)


DOCS = np.array([[0, 90, 90, 250, 300], [0, 1, 200, 201, 300]], np.int32)


@pytest.mark.parametrize("mask", ["document", "document_causal"])
@pytest.mark.parametrize("D", [128, 64])
def test_documents(mask, D):
    """Packed documents (empty and one-token ones included) on the 8-bit path; keys past
    the last boundary (Skv = 700 > 300) are in no document."""
    fa = _fa()
    B, H, Hkv, Sq, Skv = 2, 4, 2, 300, 700
    q8, k8, v8 = _inputs(B, H, Hkv, Sq, Skv, seed=106, D=D)
    scale = 1.0 / math.sqrt(D)
    o, lse = fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), scale=scale, mask_mod=mask,
                        doc_offsets=torch.from_numpy(DOCS).cuda(), score_mod="alibi")
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    _check(q8, k8, v8, o, lse, 1.0, 1.0, 1.0, scale, mask_mod=mask, doc_offsets=DOCS, score_mod="alibi")


@pytest.mark.parametrize("mask,window,offset,docs", [("causal", 0, 0, None), ("sliding_window", 200, 0, None),
                                                     ("kv_le_q_plus_offset", 0, -300, None),
                                                     ("document_causal", 0, 0, DOCS[:1])])
def test_tile_map_bit_exact(mask, window, offset, docs):
    fa = _fa()
    Sq, Skv = 640, 700
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    q8, k8, v8 = _inputs(1, 1, 1, Sq, Skv, seed=107)
    tm = torch.full((nq * nk,), 255, dtype=torch.uint8, device="cuda")
    fa.fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), mask_mod=mask, window=window, offset=offset, tile_map=tm,
               doc_offsets=None if docs is None else torch.from_numpy(docs).cuda())
    torch.cuda.synchronize()
    ref = oracle.tile_map(mask, Sq, Skv, window=window, offset=offset, doc_offsets=None if docs is None else docs[0])
    np.testing.assert_array_equal(tm.cpu().numpy().reshape(nq, nk), ref)


@pytest.mark.parametrize("mask,window,offset", [("causal", 0, 0), ("sliding_window", 300, 0),
                                                ("kv_le_q_plus_offset", 0, -100)])
def test_block_lists_from_tile_map_bitwise(mask, window, offset):
    """Lists read off the analytic tile map visit the same tiles with the same classes in
    the same order as the analytic 8-bit kernel: identical output bits."""
    fa = _fa()
    B, H, Hkv, S = 1, 4, 2, 1000
    q8, k8, v8 = (t.cuda() for t in _inputs(B, H, Hkv, S, S, seed=108))
    tm = oracle.tile_map(mask, S, S, window=window, offset=offset)
    L = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in oracle.block_mask_from_tile_map(tm, 1, 1)]
    mods = dict(mask_mod=mask, window=window, offset=offset)
    o1, l1 = fa.fwd_fp8(q8, k8, v8, **mods)
    o2, l2 = fa.fwd_fp8_block_sparse(q8, k8, v8, *L, **mods)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("mods", [dict(), dict(mask_mod="causal", score_mod="alibi"),
                                  dict(mask_mod="sliding_window", window=150)],
                         ids=["no_mod", "causal-alibi", "window150"])
def test_block_random_lists(mods):
    """Random partial / full lists (duplicates, bad indices, over-long and negative counts)
    against the oracle's block-sparse forward on the dequantized values, with the e4m3
    bound of _check computed from P of the keep matrix the lists describe."""
    from tests.helpers import random_block_lists
    from tests.test_oracle_block_pins import _dense_keep
    fa = _fa()
    B, H, Hkv, Sq, Skv, D = 2, 4, 2, 300, 700, 128
    nq, nk = -(-Sq // 128), -(-Skv // 128)
    lists = random_block_lists(np.random.default_rng(109), B, H, nq, nk, max_blocks=nk + 2, p_full=0.35, p_part=0.35)
    q8, k8, v8 = _inputs(B, H, Hkv, Sq, Skv, seed=110)
    dq, dk, dv, scale = 0.5, 2.0, 0.75, 1.0 / math.sqrt(D)
    L = [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in lists]
    o, lse = fa.fwd_fp8_block_sparse(q8.cuda(), k8.cuda(), v8.cuda(), *L, descale_q=dq, descale_k=dk, descale_v=dv,
                                     scale=scale, **mods)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = oracle.fwd_block_sparse(q8, k8, v8, *lists, scale=scale * dq * dk, **mods)
    ro = ro * dv
    # P of the keep matrix (torch float64) for the element-wise e4m3 bound
    elem = oracle.mask_matrix(mods.get("mask_mod", "none"), Sq, Skv, mods.get("window", 0)).astype(bool)
    keep = torch.from_numpy(_dense_keep(elem, *lists, B, H, Sq, Skv, 128, 128))
    qq, kk = q8.double(), k8.double().repeat_interleave(H // Hkv, 1)
    s = torch.einsum("bhid,bhjd->bhij", qq, kk) * scale * dq * dk
    if mods.get("score_mod") == "alibi":
        slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float64)
        s = s + slopes[:, None, None] * (torch.arange(Skv)[None, :] - torch.arange(Sq)[:, None]).double()
    s = s.masked_fill(~keep, float("-inf"))
    live = keep.any(-1, keepdim=True)
    P = (torch.softmax(s.masked_fill(~live, 0.0), -1) * live).numpy()
    av = np.repeat(np.abs(v8.double().numpy()), H // Hkv, axis=1)
    bound = dv * (2.0 ** -4 * np.einsum("bhij,bhjd->bhid", P, av)
                  + 2.0 ** -16 * np.einsum("bhij,bhjd->bhid", (P > 0).astype(np.float64), av))
    got = o.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ro)
    assert float((err / (1.05 * bound + 2.0 ** -8 * np.abs(ro) + 1e-4)).max()) <= 1.0
    lg = lse.cpu().numpy().astype(np.float64)
    dead = np.isneginf(rl)
    assert np.array_equal(np.isneginf(lg), dead) and np.all(got[dead] == 0.0)
    assert float(np.abs(lg[~dead] - rl[~dead]).max()) <= 1e-2
