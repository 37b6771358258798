"""GPU parity of flex_attn_decode (split-KV + combine) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.helpers import compare

pytestmark = pytest.mark.gpu

SCALE = 0.08837890625


def _fa():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    return fa


def _inputs(B, H, Hkv, cap, D, seed, dtype="f16", lens=None, mask_p=None):
    q = synth.normal_tensor((B, H, 1, D), seed * 8 + 1, dtype=dtype, device="cuda")
    kc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 2, dtype=dtype, device="cuda")
    vc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 3, dtype=dtype, device="cuda")
    kv_len = synth.kv_lengths(B, cap, seed * 8 + 4) if lens is None else torch.tensor(lens, dtype=torch.int32)
    mask = None if mask_p is None else synth.bernoulli_neg_inf_mask((B, H, 1, cap), mask_p, seed * 8 + 5, dtype=dtype)
    return q, kc, vc, kv_len, mask


def _check(q, kc, vc, kv_len, mask, scale=SCALE):
    fa = _fa()
    d = torch.device("cuda")
    o, lse = fa.decode(q.to(d), kc.to(d), vc.to(d), kv_len.to(d), scale,
                       mask=None if mask is None else mask.to(d))
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = oracle.decode(q, kc, vc, kv_len, scale, mask=mask)
    return compare(o, lse, ro, rl, "decode")


@pytest.mark.parametrize("Hkv", [32, 8])
@pytest.mark.parametrize("with_mask", [False, True])
def test_decode_config(Hkv, with_mask):
    """B=16, H=32, D=128, f16, kv_len ~ U[1, 8192], caches padded to 8192."""
    args = _inputs(16, 32, Hkv, 8192, 128, seed=3000 + Hkv, mask_p=0.1 if with_mask else None)
    _check(*args)


@pytest.mark.parametrize("Hkv", [32, 8])
def test_decode_long_kv(Hkv):
    args = _inputs(16, 32, Hkv, 8192, 128, seed=3100 + Hkv, lens=[8192] * 16, mask_p=0.1)
    _check(*args)


@pytest.mark.parametrize("lens", [[1, 255, 256, 257], [512, 0, 3, 1000], [0, 0, 0, 0]])
@pytest.mark.parametrize("D,dtype", [(128, "f16"), (64, "bf16"), (128, "bf16")])
def test_decode_split_boundaries(lens, D, dtype):
    args = _inputs(4, 8, 2, 1024, D, seed=3200 + D, dtype=dtype, lens=lens)
    _check(*args)


@pytest.mark.parametrize("H,Hkv", [(6, 2), (12, 4), (5, 5), (16, 2), (32, 2), (40, 2), (64, 4)])
def test_decode_group_sizes(H, Hkv):
    args = _inputs(3, H, Hkv, 700, 128, seed=3300 + H, mask_p=0.3)
    _check(*args)


def test_decode_all_masked_rows():
    q, kc, vc, kv_len, _ = _inputs(2, 4, 4, 300, 128, seed=3400, lens=[300, 17])
    mask = torch.zeros(2, 4, 1, 300, dtype=torch.float16, device="cuda")
    mask[0, 1] = float("-inf")
    mask[1, :, :, :17] = float("-inf")
    _check(q, kc, vc, kv_len, mask)


def test_decode_bad_kv_len_sets_status():
    fa = _fa()
    q, kc, vc, _, _ = _inputs(2, 4, 4, 64, 128, seed=3500, lens=[1, 1])
    bad = torch.tensor([65, 10], dtype=torch.int32, device="cuda")
    o, lse = fa.decode(q.cuda(), kc.cuda(), vc.cuda(), bad, SCALE)
    torch.cuda.synchronize()
    assert fa.device_status() & 1
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert fa.device_status() == 0  # cleared by the read


def test_decode_matches_forward_single_row():
    """decode(kv_len=L) == fwd(Sq=1, Skv=L) on the same data (both through the GPU)."""
    fa = _fa()
    q, kc, vc, _, _ = _inputs(1, 8, 8, 2048, 128, seed=3600, dtype="bf16", lens=[2048])
    d = torch.device("cuda")
    L = 1500
    o1, l1 = fa.decode(q.to(d), kc.to(d), vc.to(d), torch.tensor([L], dtype=torch.int32, device=d), 0.1)
    o2, l2 = fa.fwd(q.to(d), kc[:, :, :L].contiguous().to(d), vc[:, :, :L].contiguous().to(d), scale=0.1)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() < 2e-2
    assert (l1 - l2).abs().max().item() < 1e-2
