"""GPU parity of flex_attn_bwd (dQ, dK, dV) against the fp64 oracle.

The backward is named as a later phase on FlyDSL PR 931 "Add flex_attention (score_mod /
mask_mod) on the generic flash-attention kernel" (Out of scope); xformers 1094 "Tiny
upstream pr" reports mean |d - ref| of 1e-4 .. 4e-4 for its bf16 dq/dk/dv. The kernels
take the forward's O and LSE from flex_attn_fwd (as a caller would); the oracle
recomputes everything from q, k, v and dO in fp64.

Tolerances, per gradient g (bf16/f16 outputs): max |g - ref| <= 3e-2 * max |ref| and
mean |g - ref| <= 1e-2 * mean |ref| (+1e-6). P and dS enter the tensor-core products
rounded to 16 bits (relative 2^-9 / 2^-11) and the outputs are rounded once more; the
stored O (16-bit) enters delta = dO . O. Rows without keys must give exactly zero dQ.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

MAX_REL = 3e-2
MEAN_REL = 1e-2


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _check(name, got, ref):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64).reshape(g.shape)
    assert not np.isnan(g).any(), f"{name}: NaN"
    err = np.abs(g - ref)
    scale_max, scale_mean = float(np.abs(ref).max()), float(np.abs(ref).mean())
    assert err.max() <= MAX_REL * scale_max + 1e-6, f"{name}: max err {err.max():.3e} vs max|ref| {scale_max:.3e}"
    assert err.mean() <= MEAN_REL * scale_mean + 1e-6, f"{name}: mean err {err.mean():.3e} vs mean|ref| {scale_mean:.3e}"
    return float(err.mean())


def _run(q, k, v, dout, scale, **mods):
    fa = _fa()
    dev = torch.device("cuda")
    m = dict(mods)
    for key in ("alibi_slopes", "doc_offsets", "doc_offsets_kv"):
        if m.get(key) is not None:
            m[key] = torch.as_tensor(m[key]).to(dev)
    qd, kd, vd, od = (t.to(dev) for t in (q, k, v, dout))
    o, lse = fa.fwd(qd, kd, vd, scale=scale, **m)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, od, scale=scale, **m)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return dq, dk, dv


def _case(B, H, Hkv, Sq, Skv, D, dtype, seed, scale, groups=None, **mods):
    q, k, v = synth.qkv(B, H, Hkv, Sq, Skv, D, seed=seed, dtype=dtype)
    dout = synth.normal_tensor((B, H, Sq, D), seed * 8 + 7, dtype=dtype)
    dq, dk, dv = _run(q, k, v, dout, scale, **mods)
    rq, rk, rv = oracle.bwd(q, k, v, dout, scale=scale, groups=groups, **mods)
    if groups is not None:
        G = H // Hkv
        idx = [(b, hk) for b, hk in groups]
        dq = torch.stack([dq[b, hk * G:(hk + 1) * G] for b, hk in idx])
        dk = torch.stack([dk[b, hk] for b, hk in idx])
        dv = torch.stack([dv[b, hk] for b, hk in idx])
    return _check("dq", dq, rq), _check("dk", dk, rk), _check("dv", dv, rv)


def test_tiny():
    _case(1, 2, 2, 128, 128, 64, "bf16", 80, 0.125, mask_mod="causal")


MODS = [
    dict(mask_mod="none"),
    dict(mask_mod="causal"),
    dict(mask_mod="causal", score_mod="alibi"),
    dict(mask_mod="sliding_window", window=100),
    dict(mask_mod="kv_le_q_plus_offset", offset=-40),
    dict(score_mod="alibi", alibi_slopes=np.array([0.25, -0.0625, 0.5, 0.0], np.float32)),
    dict(mask_mod="document_causal", doc_offsets=np.array([[0, 90, 90, 250, 333], [0, 1, 200, 201, 300]], np.int32)),
    dict(mask_mod="document", doc_offsets=np.array([[0, 130, 131, 260, 333], [0, 64, 128, 256, 333]], np.int32)),
]


@pytest.mark.parametrize("mods", MODS, ids=lambda m: "-".join(f"{k}={v}" for k, v in m.items() if k in ("mask_mod", "score_mod")) + ("-slopes" if "alibi_slopes" in m else ""))
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f16"), (128, "f16"), (64, "bf16")])
def test_ragged_gqa(mods, D, dtype):
    _case(2, 4, 2, 333, 333, D, dtype, 81, 1.0 / math.sqrt(D), **mods)


@pytest.mark.parametrize("mods", [dict(mask_mod="none"), dict(mask_mod="causal"),
                                  dict(mask_mod="kv_le_q_plus_offset", offset=500)])
def test_cross_lengths(mods):
    """Sq != Skv, both ragged."""
    _case(1, 4, 1, 250, 1000, 128, "bf16", 82, 0.1, **mods)


def test_rows_without_keys_get_zero_dq():
    B, H, Sq, Skv, D = 1, 2, 250, 1024, 128
    q, k, v = synth.qkv(B, H, H, Sq, Skv, D, seed=83)
    dout = synth.normal_tensor((B, H, Sq, D), 84, dtype="bf16")
    mods = dict(mask_mod="kv_le_q_plus_offset", offset=-100)  # rows 0..99 keep nothing
    dq, dk, dv = _run(q, k, v, dout, 0.1, **mods)
    assert torch.all(dq[:, :, :100] == 0)
    rq, rk, rv = oracle.bwd(q, k, v, dout, scale=0.1, **mods)
    _check("dq", dq, rq), _check("dk", dk, rk), _check("dv", dv, rv)


@pytest.mark.parametrize("mods", [dict(mask_mod="none"), dict(mask_mod="causal", score_mod="alibi"),
                                  dict(mask_mod="sliding_window", window=256)])
def test_mha_2048_sampled_groups(mods):
    """B=2, H=32, S=2048, D=128; the oracle computes two (b, head) groups in full."""
    _case(2, 32, 32, 2048, 2048, 128, "bf16", 85, 1.0 / math.sqrt(128), groups=[(0, 3), (1, 31)], **mods)


def test_gqa_4096_sampled_group():
    _case(1, 8, 2, 4096, 4096, 128, "bf16", 86, 1.0 / math.sqrt(128), groups=[(0, 1)], mask_mod="causal")


@pytest.mark.parametrize("dtype,mods", [("bf16", dict(mask_mod="none")), ("f16", dict(mask_mod="causal")),
                                        ("bf16", dict(mask_mod="sliding_window", window=300))])
def test_d64_ring_wrap_sampled_group(dtype, mods):
    """D=64 at Sq = Skv = 1500: 12 key tiles (ragged), so both of the dQ kernel's key and
    value rings and the dK/dV kernel's query ring wrap several times."""
    _case(1, 4, 2, 1500, 1500, 64, dtype, 87, 0.125, groups=[(0, 1)], **mods)


@pytest.mark.parametrize("mods", [dict(mask_mod="none"), dict(mask_mod="causal")], ids=["no_mod", "causal"])
def test_long_8192_sampled_groups(mods):
    """The size the bench times: B2 H32 S8192 D128 bf16 with the bench's inputs
    (N(0, 0.5^2), dO ~ N(0, 1)); the oracle computes two whole (b, head) groups, the
    first and the last, in full."""
    fa = _fa()
    B, H, S, D = 2, 32, 8192, 128
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=4000, sigma=0.5, device="cuda")
    dout = synth.normal_tensor((B, H, S, D), 4103, dtype="bf16", device="cuda")
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = _run(q, k, v, dout, scale, **mods)
    groups = [(0, 0), (1, 31)]
    rq, rk, rv = oracle.bwd(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), scale=scale, groups=groups, **mods)
    dq = torch.stack([dq[b, hk:hk + 1] for b, hk in groups])
    dk = torch.stack([dk[b, hk] for b, hk in groups])
    dv = torch.stack([dv[b, hk] for b, hk in groups])
    _check("dq", dq, rq), _check("dk", dk, rk), _check("dv", dv, rv)
