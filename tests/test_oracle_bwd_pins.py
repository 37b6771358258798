"""Pins for the oracle's backward pass (dQ, dK, dV of sum(dO * O)).

The backward is named as a later phase on FlyDSL PR 931 "Add flex_attention (score_mod /
mask_mod) on the generic flash-attention kernel" (Out of scope); xformers 1094 "Tiny
upstream pr" reports mean dq/dk/dv errors of a backward against a reference. The oracle
restates the gradient of the forward's definition; these tests check it against:
  * torch float64 autograd through an explicit masked softmax (a library special case),
  * central finite differences of the oracle's own forward on inputs where the step is
    exact in bf16 (pins the gradient to the function, not to a formula),
  * closed forms: one key (P = 1, so dQ = dK = 0 and dV sums dO), fully masked rows,
  * the shift invariance: adding one vector to every key changes no gradient.
"""
import numpy as np
import pytest
import torch

import synth

TOL = 1e-12


def _autograd(q, k, v, dout, scale, keep=None, slopes=None):
    B, H, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    qq, kk, vv = (t.double().requires_grad_() for t in (q, k, v))
    G = H // Hkv
    s = torch.einsum("bhid,bhjd->bhij", qq, kk.repeat_interleave(G, 1)) * scale
    if slopes is not None:
        rel = (torch.arange(Skv)[None, :] - torch.arange(Sq)[:, None]).double()
        s = s + torch.as_tensor(slopes, dtype=torch.float64)[:, None, None] * rel
    if keep is not None:
        kt = torch.from_numpy(np.broadcast_to(keep, (B, H, Sq, Skv)).copy())
        s = s.masked_fill(~kt, float("-inf"))
        live = kt.any(-1, keepdim=True)
        s = s.masked_fill(~live, 0.0)
        p = torch.softmax(s, -1) * live
    else:
        p = torch.softmax(s, -1)
    o = p @ vv.repeat_interleave(G, 1)
    (o * dout.double()).sum().backward()
    return qq.grad.numpy(), kk.grad.numpy(), vv.grad.numpy()


def _slopes(H):
    return [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]


@pytest.mark.parametrize("mask,window,offset", [("none", 0, 0), ("causal", 0, 0), ("sliding_window", 4, 0),
                                                ("kv_le_q_plus_offset", 0, -6)])
@pytest.mark.parametrize("score", ["none", "alibi"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_bwd_equals_torch_autograd(oracle_mod, mask, window, offset, score, dtype):
    B, H, Hkv, Sq, Skv, D = 2, 4, 2, 11, 15, 8
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=61, dtype=dtype)
    dout = synth.normal_tensor((B, H, Sq, D), 62, dtype="bf16" if dtype == torch.bfloat16 else "f16")
    dq, dk, dv = oracle_mod.bwd(q, k, v, dout, scale=0.35, score_mod=score, mask_mod=mask, window=window,
                                offset=offset)
    keep = oracle_mod.mask_matrix(mask, Sq, Skv, window, offset).astype(bool)
    rq, rk, rv = _autograd(q, k, v, dout, 0.35, keep=keep, slopes=_slopes(H) if score == "alibi" else None)
    np.testing.assert_allclose(dq, rq, atol=TOL, rtol=0)
    np.testing.assert_allclose(dk, rk, atol=TOL, rtol=0)
    np.testing.assert_allclose(dv, rv, atol=TOL, rtol=0)


def test_bwd_documents_and_slope_table_equal_autograd(oracle_mod):
    B, H, Hkv, S, D = 2, 2, 1, 20, 8
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=63)
    dout = synth.normal_tensor((B, H, S, D), 64, dtype="bf16")
    off = np.array([[0, 7, 7, 16, 20], [0, 1, 12, 18, 18]], np.int32)
    table = [0.5, -0.125]
    dq, dk, dv = oracle_mod.bwd(q, k, v, dout, scale=0.4, score_mod="alibi", mask_mod="document_causal",
                                doc_offsets=off, alibi_slopes=table)
    keep = np.stack([oracle_mod.mask_matrix("document_causal", S, S, doc_offsets=off[b]) for b in range(B)])
    rq, rk, rv = _autograd(q, k, v, dout, 0.4, keep=keep[:, None].astype(bool), slopes=table)
    np.testing.assert_allclose(dq, rq, atol=TOL, rtol=0)
    np.testing.assert_allclose(dk, rk, atol=TOL, rtol=0)
    np.testing.assert_allclose(dv, rv, atol=TOL, rtol=0)


def test_bwd_group_subset_equals_full(oracle_mod):
    B, H, Hkv, Sq, Skv, D = 2, 6, 3, 9, 10, 8
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=65)
    dout = synth.normal_tensor((B, H, Sq, D), 66, dtype="bf16")
    dq, dk, dv = oracle_mod.bwd(q, k, v, dout, scale=0.3, mask_mod="causal")
    sq, sk, sv = oracle_mod.bwd(q, k, v, dout, scale=0.3, mask_mod="causal", groups=[(1, 2), (0, 0)])
    np.testing.assert_array_equal(sq[0], dq[1, 4:6])
    np.testing.assert_array_equal(sk[0], dk[1, 2])
    np.testing.assert_array_equal(sv[1], dv[0, 0])


def _grid_inputs(B, H, S, D, seed):
    """Values on a grid of 1/8 in [-1, 1): q +- 2^-7 and k + 1/8 stay exact in bf16."""
    rng = np.random.default_rng(seed)
    mk = lambda: torch.tensor(rng.integers(-8, 8, (B, H, S, D)) / 8.0, dtype=torch.float64)
    return mk(), mk(), mk(), mk()


def test_bwd_equals_finite_differences_of_forward(oracle_mod):
    B, H, S, D = 1, 1, 6, 4
    q, k, v, dout = (t.to(torch.bfloat16) for t in _grid_inputs(B, H, S, D, 67))
    h = 2.0 ** -7
    scale = 0.5
    dq, dk, dv = oracle_mod.bwd(q, k, v, dout, scale=scale, mask_mod="causal")

    def loss(q_, k_, v_):
        o, _ = oracle_mod.fwd(q_, k_, v_, scale=scale, mask_mod="causal")
        return float((o * dout.double().numpy()).sum())
    for name, t, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 1, 2), (0, 0, 4, 0), (0, 0, 5, 3), (0, 0, 2, 1)]:
            plus, minus = t.clone(), t.clone()
            plus[idx] = (t[idx].double() + h).to(torch.bfloat16)
            minus[idx] = (t[idx].double() - h).to(torch.bfloat16)
            assert float(plus[idx]) - float(minus[idx]) == 2 * h  # exact steps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            lp = loss(*[plus if a is t else a for a in args])
            lm = loss(*[minus if a is t else a for a in args])
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[idx]) <= 2e-4 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])


def test_bwd_single_key_closed_form(oracle_mod):
    B, H, Hkv, Sq, D = 1, 4, 2, 5, 8
    q, k, v = synth.qkv(B, H, Hkv, Sq, 1, D, seed=68)
    dout = synth.normal_tensor((B, H, Sq, D), 69, dtype="bf16")
    dq, dk, dv = oracle_mod.bwd(q, k, v, dout, scale=0.7)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)
    want = dout.double().numpy().reshape(B, Hkv, 2, Sq, D).sum(axis=(2, 3))
    np.testing.assert_allclose(dv[:, :, 0, :], want, atol=TOL, rtol=0)


def test_bwd_fully_masked_rows_have_no_gradient(oracle_mod):
    B, H, Sq, Skv, D = 1, 2, 8, 8, 8
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=70)
    dout = synth.normal_tensor((B, H, Sq, D), 71, dtype="bf16")
    # kv <= q - 3: rows 0..2 keep nothing
    dq, dk, dv = oracle_mod.bwd(q, k, v, dout, scale=0.5, mask_mod="kv_le_q_plus_offset", offset=-3)
    assert np.all(dq[:, :, :3] == 0.0)
    # and changing dO on those rows changes nothing
    d2 = dout.clone()
    d2[:, :, :3] = 5.0
    dq2, dk2, dv2 = oracle_mod.bwd(q, k, v, d2, scale=0.5, mask_mod="kv_le_q_plus_offset", offset=-3)
    np.testing.assert_array_equal(dq, dq2)
    np.testing.assert_array_equal(dk, dk2)
    np.testing.assert_array_equal(dv, dv2)


def test_bwd_key_shift_invariance(oracle_mod):
    B, H, S, D = 1, 2, 9, 8
    q, k, v, dout = (t.to(torch.bfloat16) for t in _grid_inputs(B, H, S, D, 72))
    c = torch.tensor(np.random.default_rng(73).integers(-4, 4, D) / 8.0, dtype=torch.float64)
    k2 = (k.double() + c).to(torch.bfloat16)
    assert torch.equal(k2.double(), k.double() + c)  # exact
    g1 = oracle_mod.bwd(q, k, v, dout, scale=0.5, mask_mod="causal")
    g2 = oracle_mod.bwd(q, k2, v, dout, scale=0.5, mask_mod="causal")
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)
