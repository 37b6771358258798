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


def _check(q, kc, vc, kv_len, mask, scale=SCALE, split=0):
    fa = _fa()
    d = torch.device("cuda")
    o, lse = fa.decode(q.to(d), kc.to(d), vc.to(d), kv_len.to(d), scale,
                       mask=None if mask is None else mask.to(d), split_size=split)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    ro, rl = oracle.decode(q, kc, vc, kv_len, scale, mask=mask)
    return compare(o, lse, ro, rl, "decode")


@pytest.mark.parametrize("Hkv", [32, 8])
@pytest.mark.parametrize("with_mask", [False, True])
@pytest.mark.parametrize("split", [0, 128, 256])
def test_decode_config(Hkv, with_mask, split):
    """B=16, H=32, D=128, f16, kv_len ~ U[1, 8192], caches padded to 8192; the library's
    split size and both explicit ones, every row against the oracle."""
    args = _inputs(16, 32, Hkv, 8192, 128, seed=3000 + Hkv, mask_p=0.1 if with_mask else None)
    _check(*args, split=split)


@pytest.mark.parametrize("Hkv", [32, 8])
def test_decode_long_kv(Hkv):
    args = _inputs(16, 32, Hkv, 8192, 128, seed=3100 + Hkv, lens=[8192] * 16, mask_p=0.1)
    _check(*args)


@pytest.mark.parametrize("lens", [[1, 255, 256, 257], [512, 0, 3, 1000], [0, 0, 0, 0], [127, 128, 129, 383]])
@pytest.mark.parametrize("D,dtype", [(128, "f16"), (64, "bf16"), (128, "bf16")])
@pytest.mark.parametrize("split", [128, 256])
def test_decode_split_boundaries(lens, D, dtype, split):
    args = _inputs(4, 8, 2, 1024, D, seed=3200 + D, dtype=dtype, lens=lens)
    _check(*args, split=split)
    args = _inputs(4, 8, 8, 1024, D, seed=3250 + D, dtype=dtype, lens=lens)  # one query head per kv head
    _check(*args, split=split)


@pytest.mark.parametrize("Hkv", [32, 8])
def test_decode_split_size_independence(Hkv):
    """The combine merges chunk partials exactly in real arithmetic, so 128- and
    256-position splits give the same rows up to rounding: both against the oracle and
    against each other (O within 4e-3, LSE within 1e-3)."""
    fa = _fa()
    q, kc, vc, kv_len, mask = _inputs(16, 32, Hkv, 8192, 128, seed=3700 + Hkv, mask_p=0.1)
    d = torch.device("cuda")
    args = (q.to(d), kc.to(d), vc.to(d), kv_len.to(d), SCALE)
    o1, l1 = fa.decode(*args, mask=mask.to(d), split_size=128)
    o2, l2 = fa.decode(*args, mask=mask.to(d), split_size=256)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, kc, vc, kv_len, SCALE, mask=mask)
    compare(o1, l1, ro, rl, "split 128")
    compare(o2, l2, ro, rl, "split 256")
    assert torch.equal(torch.isneginf(l1), torch.isneginf(l2))
    fin = ~torch.isneginf(l1)
    assert (o1.float() - o2.float()).abs().max().item() <= 4e-3
    assert (l1[fin] - l2[fin]).abs().max().item() <= 1e-3


@pytest.mark.parametrize("H,Hkv", [(6, 2), (12, 4), (5, 5), (16, 2), (32, 2), (40, 2), (64, 4)])
@pytest.mark.parametrize("cap", [700, 704])
def test_decode_group_sizes(H, Hkv, cap):
    """Grouped heads: 2..20 query heads per kv head (up to two 16-row groups).  cap = 704
    streams the mask tiles with TMA, cap = 700 (rows not a multiple of 16 bytes) reads them
    directly."""
    args = _inputs(3, H, Hkv, cap, 128, seed=3300 + H, mask_p=0.3)
    _check(*args)


def test_decode_large_batch():
    """B above the grouped-query kernel's batch table (1024): the register-streaming kernel."""
    args = _inputs(1030, 4, 2, 64, 64, seed=3350, dtype="bf16", mask_p=0.2)
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


def test_decode_per_call_status_on_two_streams():
    """A bad kv_len on one stream and a clean decode on another, each with its own status
    word: only the first caller's word gets bit 1, and the shared word stays clear."""
    fa = _fa()
    assert fa.device_status() == 0
    q, kc, vc, _, _ = _inputs(2, 8, 2, 512, 128, seed=3550, lens=[1, 1])
    q, kc, vc = q.cuda(), kc.cuda(), vc.cuda()
    bad = torch.tensor([513, 100], dtype=torch.int32, device="cuda")
    good = torch.tensor([512, 100], dtype=torch.int32, device="cuda")
    st_a = torch.zeros(1, dtype=torch.int32, device="cuda")
    st_b = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(sa):
        oa, la = fa.decode(q, kc, vc, bad, SCALE, status=st_a)
    with torch.cuda.stream(sb):
        ob, lb = fa.decode(q, kc, vc, good, SCALE, status=st_b)
        fwd_st = torch.zeros(1, dtype=torch.int32, device="cuda")
        fa.fwd(q, kc, vc, status=fwd_st)
    torch.cuda.synchronize()
    assert int(st_a.item()) == 1
    assert int(st_b.item()) == 0 and int(fwd_st.item()) == 0
    assert fa.device_status() == 0
    assert torch.all(oa[0] == 0) and torch.all(torch.isneginf(la[0]))
    ro, rl = oracle.decode(q.cpu(), kc.cpu(), vc.cpu(), good.cpu(), SCALE)
    compare(ob, lb, ro, rl, "clean stream")


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


def test_decode_grouped_graph_replay():
    """A CUDA graph of a grouped-query decode (the persistent kernel and the combine):
    each replay, with new lengths written into the captured kv_len tensor, equals an
    eager call, because the chunk list is built on the device from kv_len."""
    fa = _fa()
    B, H, Hkv, cap, D = 4, 16, 4, 2048, 128
    q, kc, vc, _, mask = _inputs(B, H, Hkv, cap, D, seed=3800, lens=[1] * B, mask_p=0.1)
    d = torch.device("cuda")
    q, kc, vc, mask = q.to(d), kc.to(d), vc.to(d), mask.to(d)
    kv_len = torch.full((B,), cap, dtype=torch.int32, device=d)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=d)
    ws = torch.empty(fa.decode_workspace_size(B, H, Hkv, cap, D), dtype=torch.uint8, device=d)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fa.decode(q, kc, vc, kv_len, SCALE, mask=mask, out=out, lse_out=lse, workspace=ws)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fa.decode(q, kc, vc, kv_len, SCALE, mask=mask, out=out, lse_out=lse, workspace=ws)
    for lens in ([cap, 1, 700, 1500], [0, 2048, 64, 65], [1000, 1000, 1000, 1000]):
        kv_len.copy_(torch.tensor(lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        ref_o, ref_l = fa.decode(q, kc, vc, kv_len, SCALE, mask=mask)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l), lens
    assert fa.device_status() == 0
