"""Pins for the fp64 oracle, checked against things other than itself.

Each test pins the oracle to a closed form, an exact identity of the method,
a library special case (torch float64 softmax / logsumexp on CPU), or a value
printed on the source pages (fixtures under tests/golden/).  Chosen so that a
plausible slip in the oracle -- dropped scale, sign of the alibi bias, slope
index, off-by-one in a mask, GQA head mapping, LSE base, NaN on fully masked
rows, decode length handling, mask-vs-scale order -- fails at least one.
"""
import math
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def _t(vals, dtype=torch.bfloat16):
    return torch.tensor(vals, dtype=torch.float64).to(dtype)


# ---------------------------------------------------------------- library special case

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_no_mod_equals_torch_float64_softmax(oracle_mod, dtype):
    """no_mod is plain SDPA: softmax(scale Q K^T) V and logsumexp (torch, fp64, CPU)."""
    B, H, Sq, Skv, D = 2, 3, 17, 23, 8
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=11, dtype=dtype)
    scale = 0.37
    o, lse = oracle_mod.fwd(q, k, v, scale=scale)
    s = torch.einsum("bhid,bhjd->bhij", q.double(), k.double()) * scale
    ref_o = torch.softmax(s, dim=-1) @ v.double()
    ref_lse = torch.logsumexp(s, dim=-1)
    np.testing.assert_allclose(o, ref_o.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def test_causal_equals_torch_masked_softmax(oracle_mod):
    """causal_via_mask == softmax with an explicit lower-triangular boolean mask."""
    B, H, S, D = 1, 2, 19, 8
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=12)
    o, lse = oracle_mod.fwd(q, k, v, scale=0.5, mask_mod="causal")
    s = torch.einsum("bhid,bhjd->bhij", q.double(), k.double()) * 0.5
    keep = torch.ones(S, S, dtype=torch.bool).tril()
    s = s.masked_fill(~keep, float("-inf"))
    np.testing.assert_allclose(o, (torch.softmax(s, -1) @ v.double()).numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12, rtol=0)


# ---------------------------------------------------------------- hand-worked closed forms

def test_two_keys_closed_form(oracle_mod):
    q = _t([2.0]).reshape(1, 1, 1, 1)
    k = _t([1.0, 0.0]).reshape(1, 1, 2, 1)
    v = _t([3.0, 5.0]).reshape(1, 1, 2, 1)
    o, lse = oracle_mod.fwd(q, k, v, scale=0.5)
    e = math.e
    assert abs(o[0, 0, 0, 0] - (3 * e + 5) / (e + 1)) < TOL
    assert abs(lse[0, 0, 0] - math.log(e + 1)) < TOL


def test_scale_then_alibi_order_and_slopes(oracle_mod):
    """score_mod sees the already scaled score; slope_h = 2^(-8(h+1)/H)."""
    H = 8
    q = _t([2.0] * H).reshape(1, H, 1, 1)
    k = _t([1.0, 0.0] * H).reshape(1, H, 2, 1)
    v = _t([3.0, 5.0] * H).reshape(1, H, 2, 1)
    o, lse = oracle_mod.fwd(q, k, v, scale=0.5, score_mod="alibi")
    for h in range(H):
        s = 2.0 ** (-(h + 1))          # 2^(-8(h+1)/8)
        assert oracle_mod.alibi_slope(h, H) == s
        w0, w1 = math.exp(1.0), math.exp(s)   # x = [1 + s*0, 0 + s*1]
        assert abs(o[0, h, 0, 0] - (3 * w0 + 5 * w1) / (w0 + w1)) < TOL
        assert abs(lse[0, h, 0] - math.log(w0 + w1)) < TOL


@pytest.mark.parametrize("mask,window,offset", [
    ("causal", 0, 0), ("sliding_window", 5, 0), ("sliding_window", 1, 0),
    ("kv_le_q_plus_offset", 0, 3), ("kv_le_q_plus_offset", 0, -4)])
def test_zero_query_counts(oracle_mod, mask, window, offset):
    """Q = 0: O = mean of the kept V rows, LSE = ln(count); count is a closed form."""
    S, D = 13, 4
    q = torch.zeros(1, 1, S, D, dtype=torch.bfloat16)
    k = synth.normal_tensor((1, 1, S, D), 5)
    v = synth.normal_tensor((1, 1, S, D), 6)
    o, lse = oracle_mod.fwd(q, k, v, scale=0.3, mask_mod=mask, window=window, offset=offset)
    vd = v.double().numpy()[0, 0]
    for i in range(S):
        if mask == "causal":
            lo, hi = 0, i + 1
        elif mask == "sliding_window":
            lo, hi = max(0, i - window + 1), i + 1
        else:
            lo, hi = 0, max(0, min(S, i + offset + 1))
        cnt = hi - lo
        if cnt == 0:
            assert lse[0, 0, i] == -np.inf and np.all(o[0, 0, i] == 0.0)
        else:
            assert abs(lse[0, 0, i] - math.log(cnt)) < TOL
            np.testing.assert_allclose(o[0, 0, i], vd[lo:hi].mean(0), atol=1e-12, rtol=0)


@pytest.mark.parametrize("H,h", [(4, 0), (4, 3), (32, 0), (32, 7)])
def test_alibi_zero_query_closed_form(oracle_mod, H, h):
    """Q = 0, alibi: LSE_i = -s i + ln((e^{sN}-1)/(e^s-1)); V[j,0]=j gives the mean of j."""
    N, D = 200, 2
    q = torch.zeros(1, H, N, D, dtype=torch.bfloat16)
    k = synth.normal_tensor((1, H, N, D), 7)
    v = torch.zeros(1, H, N, D, dtype=torch.float64)
    v[..., 0] = torch.arange(N, dtype=torch.float64)
    v[..., 1] = 1.0
    v = v.to(torch.bfloat16)
    o, lse = oracle_mod.fwd(q, k, v, scale=1.0, score_mod="alibi")
    s = 2.0 ** (-8.0 * (h + 1) / H)
    base = math.log((math.exp(s * N) - 1.0) / (math.exp(s) - 1.0))
    mean_j = N * math.exp(s * N) / (math.exp(s * N) - 1.0) - math.exp(s) / (math.exp(s) - 1.0)
    for i in (0, 1, 57, N - 1):
        assert abs(lse[0, h, i] - (-s * i + base)) < 1e-9
        assert abs(o[0, h, i, 0] - mean_j) < 1e-9
        assert abs(o[0, h, i, 1] - 1.0) < 1e-12


# ---------------------------------------------------------------- exact identities

def test_identities_between_masks(oracle_mod):
    B, H, S, D = 1, 2, 40, 8
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=21)
    run = lambda **kw: oracle_mod.fwd(q, k, v, scale=0.25, **kw)
    o0, l0 = run()
    # an all-true mask (kv <= q + Skv) is no_mod
    o1, l1 = run(mask_mod="kv_le_q_plus_offset", offset=S)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    # kv <= q + 0 is causal; a window at least as long as the sequence is causal
    oc, lc = run(mask_mod="causal")
    o2, l2 = run(mask_mod="kv_le_q_plus_offset", offset=0)
    o3, l3 = run(mask_mod="sliding_window", window=S)
    assert np.array_equal(oc, o2) and np.array_equal(lc, l2)
    assert np.array_equal(oc, o3) and np.array_equal(lc, l3)
    # causal_fast (causal=True) keeps exactly the same pairs
    o4, l4 = run(mask_mod="causal_fast")
    assert np.array_equal(oc, o4) and np.array_equal(lc, l4)
    # first causal row attends to key 0 only
    np.testing.assert_array_equal(oc[0, :, 0], v.double().numpy()[0, :, 0])


def test_probabilities_sum_to_one(oracle_mod):
    q, k, v = synth.qkv(1, 3, 3, 9, 31, 8, seed=22)
    for kw in ({}, {"mask_mod": "causal"}, {"score_mod": "alibi", "mask_mod": "sliding_window", "window": 4}):
        _, _, p = oracle_mod.fwd(q, k, v, scale=0.4, want_probs=True, **kw)
        np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12, rtol=0)
        assert np.all(p >= 0)


def test_gqa_equals_repeated_kv(oracle_mod):
    """GQA(H, Hkv) == MHA with K/V repeat_interleaved G times (query head h reads h // G)."""
    B, H, Hkv, Sq, Skv, D = 2, 8, 2, 11, 14, 8
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=23)
    G = H // Hkv
    for kw in ({}, {"score_mod": "alibi", "mask_mod": "causal"}):
        o, l = oracle_mod.fwd(q, k, v, scale=0.3, **kw)
        o2, l2 = oracle_mod.fwd(q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1), scale=0.3, **kw)
        assert np.array_equal(o, o2) and np.array_equal(l, l2)
    # and not the other plausible mapping h % Hkv
    o3, _ = oracle_mod.fwd(q, k.repeat(1, G, 1, 1), v.repeat(1, G, 1, 1), scale=0.3)
    o, _ = oracle_mod.fwd(q, k, v, scale=0.3)
    assert not np.allclose(o, o3)


def test_alibi_row_shift(oracle_mod):
    """With Q = 0 the alibi bias of row i is row 0's minus s*i: O is the same, LSE shifts."""
    H, N = 4, 64
    q = torch.zeros(1, H, N, 8, dtype=torch.bfloat16)
    k = synth.normal_tensor((1, H, N, 8), 31)
    v = synth.normal_tensor((1, H, N, 8), 32)
    o, lse = oracle_mod.fwd(q, k, v, score_mod="alibi")
    for h in range(H):
        s = 2.0 ** (-8.0 * (h + 1) / H)
        np.testing.assert_allclose(o[0, h], np.broadcast_to(o[0, h, :1], o[0, h].shape), atol=1e-12)
        np.testing.assert_allclose(lse[0, h] - lse[0, h, 0], -s * np.arange(N), atol=1e-10)


def test_row_subset_matches_full(oracle_mod):
    q, k, v = synth.qkv(2, 4, 2, 33, 40, 16, seed=24)
    o, l = oracle_mod.fwd(q, k, v, score_mod="alibi", mask_mod="sliding_window", window=7)
    rows = np.array([0, 5, 32, 33, 2 * 4 * 33 - 1, 100], dtype=np.int64)
    os_, ls = oracle_mod.fwd(q, k, v, score_mod="alibi", mask_mod="sliding_window", window=7, rows=rows)
    assert np.array_equal(os_, o.reshape(-1, 16)[rows]) and np.array_equal(ls, l.reshape(-1)[rows])


# ---------------------------------------------------------------- fully masked rows

def test_cross_attention_fully_masked(oracle_mod):
    """Sq=250, Skv=1024, keep kv <= q - 300: every row is fully masked -> O = 0, LSE = -inf."""
    q, k, v = synth.qkv(1, 2, 1, 250, 1024, 16, seed=25)
    o, lse = oracle_mod.fwd(q, k, v, mask_mod="kv_le_q_plus_offset", offset=-300)
    assert np.all(o == 0.0) and not np.any(np.signbit(o))
    assert np.all(lse == -np.inf)
    # a partly masked variant: rows i < 300 - ... none kept until i >= 300 - offset
    o2, l2 = oracle_mod.fwd(q, k, v, mask_mod="kv_le_q_plus_offset", offset=-100)
    assert np.all(l2[..., :100] == -np.inf) and np.all(np.isfinite(l2[..., 100:]))
    assert not np.any(np.isnan(o2))


# ---------------------------------------------------------------- decode

def test_decode_equals_forward_single_row(oracle_mod):
    B, H, Hkv, cap, D = 3, 4, 2, 50, 16
    q = synth.normal_tensor((B, H, 1, D), 41, dtype="f16")
    kc = synth.normal_tensor((B, Hkv, cap, D), 42, dtype="f16")
    vc = synth.normal_tensor((B, Hkv, cap, D), 43, dtype="f16")
    lens = torch.tensor([1, 37, 50], dtype=torch.int32)
    o, lse = oracle_mod.decode(q, kc, vc, lens, scale=0.08837890625)
    for b in range(B):
        L = int(lens[b])
        of, lf = oracle_mod.fwd(q[b:b + 1], kc[b:b + 1, :, :L], vc[b:b + 1, :, :L], scale=0.08837890625)
        np.testing.assert_allclose(o[b], of[0], atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse[b], lf[0], atol=1e-13, rtol=0)


def test_decode_mask_cutoff_equals_shorter_length(oracle_mod):
    B, H, cap, D = 2, 2, 40, 8
    q = synth.normal_tensor((B, H, 1, D), 44, dtype="f16")
    kc = synth.normal_tensor((B, H, cap, D), 45, dtype="f16")
    vc = synth.normal_tensor((B, H, cap, D), 46, dtype="f16")
    full = torch.tensor([40, 40], dtype=torch.int32)
    mask = torch.zeros(B, H, 1, cap, dtype=torch.float16)
    mask[..., 23:] = float("-inf")
    o1, l1 = oracle_mod.decode(q, kc, vc, full, 0.3, mask=mask)
    o2, l2 = oracle_mod.decode(q, kc, vc, torch.tensor([23, 23], dtype=torch.int32), 0.3)
    np.testing.assert_allclose(o1, o2, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-13, rtol=0)


def test_decode_empty_and_all_masked(oracle_mod):
    B, H, cap, D = 2, 2, 16, 8
    q = synth.normal_tensor((B, H, 1, D), 47, dtype="f16")
    kc = synth.normal_tensor((B, H, cap, D), 48, dtype="f16")
    vc = synth.normal_tensor((B, H, cap, D), 49, dtype="f16")
    o, l = oracle_mod.decode(q, kc, vc, torch.tensor([0, 5], dtype=torch.int32), 0.3)
    assert np.all(o[0] == 0) and np.all(l[0] == -np.inf) and np.all(np.isfinite(l[1]))
    mask = torch.full((B, H, 1, cap), float("-inf"), dtype=torch.float16)
    o, l = oracle_mod.decode(q, kc, vc, torch.tensor([16, 16], dtype=torch.int32), 0.3, mask=mask)
    assert np.all(o == 0) and np.all(l == -np.inf)


@pytest.mark.parametrize("L", [1, 7, 60])
def test_decode_finite_mask_added_after_scale(oracle_mod, L):
    """q = 0 and mask m_j = j/4: weights e^{j/4}; closed form (hand_worked.md item 5)."""
    cap, D = 64, 2
    q = torch.zeros(1, 1, 1, D, dtype=torch.float16)
    kc = synth.normal_tensor((1, 1, cap, D), 50, dtype="f16")
    vc = torch.zeros(1, 1, cap, D, dtype=torch.float64)
    vc[..., 0] = torch.arange(cap, dtype=torch.float64)
    vc[..., 1] = 1.0
    vc = vc.half()
    mask = (torch.arange(cap, dtype=torch.float64) / 4).reshape(1, 1, 1, cap).half()
    o, lse = oracle_mod.decode(q, kc, vc, torch.tensor([L], dtype=torch.int32), 0.08837890625, mask=mask)
    s = 0.25
    if L == 1:
        exp_lse, exp_mean = 0.0, 0.0
    else:
        exp_lse = math.log((math.exp(s * L) - 1) / (math.exp(s) - 1))
        exp_mean = L * math.exp(s * L) / (math.exp(s * L) - 1) - math.exp(s) / (math.exp(s) - 1)
    assert abs(lse[0, 0, 0] - exp_lse) < 1e-9
    assert abs(o[0, 0, 0, 0] - exp_mean) < 1e-9
    assert abs(o[0, 0, 0, 1] - 1.0) < 1e-12


# ---------------------------------------------------------------- tile map / element mask

def test_tile_map_closed_forms(oracle_mod):
    c = oracle_mod.tile_map("causal", 384, 384)
    np.testing.assert_array_equal(c, [[2, 0, 0], [1, 2, 0], [1, 1, 2]])
    n = oracle_mod.tile_map("none", 250, 250)        # pad tail is PARTIAL
    np.testing.assert_array_equal(n, [[1, 2], [1, 2]])
    n = oracle_mod.tile_map("none", 300, 256)
    np.testing.assert_array_equal(n, [[1, 1]] * 3)
    # sliding window of 256 keys at S=640: diagonal PARTIAL, one FULL tile before it,
    # then PARTIAL (the lower edge of the band), EMPTY beyond
    w = oracle_mod.tile_map("sliding_window", 640, 640, window=256)
    exp = np.zeros((5, 5), dtype=np.uint8)
    for t in range(5):
        exp[t, t] = 2
        if t >= 1:
            exp[t, t - 1] = 1
        if t >= 2:
            exp[t, t - 2] = 2
    np.testing.assert_array_equal(w, exp)
    x = oracle_mod.tile_map("kv_le_q_plus_offset", 250, 1024, offset=-300)
    assert x.shape == (2, 8) and np.all(x == 0)


def test_mask_matrix_counts(oracle_mod):
    S = 50
    assert oracle_mod.mask_matrix("causal", S, S).sum() == S * (S + 1) // 2
    W = 7
    assert oracle_mod.mask_matrix("sliding_window", S, S, window=W).sum() == sum(min(i + 1, W) for i in range(S))
    assert oracle_mod.mask_matrix("none", 3, 5).sum() == 15
    m = oracle_mod.mask_matrix("kv_le_q_plus_offset", 4, 6, offset=1)
    np.testing.assert_array_equal(m.sum(1), [2, 3, 4, 5])


# ---------------------------------------------------------------- page-printed values

def _perf_rows():
    rows = []
    with open(os.path.join(GOLDEN, "flydsl_mi300x_perf_table.tsv")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            S, case, lat, tf, counting = line.split("\t")
            rows.append((int(S), case, float(lat), float(tf), counting.strip()))
    return rows


def test_flop_count_reproduces_printed_tflops(oracle_mod):
    """4*B*H*S^2*D / latency reproduces every printed TFLOPS (B=2, H=32, D=128)."""
    rows = _perf_rows()
    assert len(rows) == 27
    for S, case, lat, tf, counting in rows:
        flops = oracle_mod.fwd_flops(2, 32, S, S, 128) * (0.5 if counting == "half" else 1.0)
        got = flops / (lat * 1e-6) / 1e12
        assert abs(got - tf) / tf < 2e-3, (S, case, got, tf)


def test_decode_scale_is_f16_of_inv_sqrt_d():
    """The decode example's scale constant 8.837890e-02 : f16 is f16(1/sqrt(128))."""
    with open(os.path.join(GOLDEN, "iree_decode_example.txt")) as f:
        vals = dict(l.split("\t")[:2] for l in f if not l.startswith("#") and "\t" in l)
    printed = float(vals["scale"])
    as_f16 = float(torch.tensor(printed, dtype=torch.float64).half())
    assert as_f16 == 0.08837890625 == float(torch.tensor(1 / math.sqrt(128)).half())
    assert vals["q"] == "1x32x1x128"
