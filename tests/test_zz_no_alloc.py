"""flex_attn_decode_noalloc: the decode entry point for callers that cannot allocate.

Hosts that pass only inputs and outputs, processes whose device memory budget is
already reserved, and decode loops that cannot afford the device-wide synchronisation
of cudaMalloc/cudaFree call this variant; its scratch lives in an array compiled into
the library.  This test calls it through the C ABI twice in a row (with different
inputs, so the second call runs over the first call's leftover scratch) and checks
each result against flex_attn_decode with a caller-allocated workspace, within the
parity tolerances of the other decode tests.  It also checks that a size whose
workspace exceeds the compiled-in limit is refused.  Kept in a file of its own so that
pytest collects it last.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

SCALE = 0.08837890625


def _inputs(B, H, Hkv, cap, D, seed, lens):
    q = synth.normal_tensor((B, H, 1, D), seed * 8 + 1, dtype="f16", device="cuda")
    kc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 2, dtype="f16", device="cuda")
    vc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 3, dtype="f16", device="cuda")
    mask = synth.bernoulli_neg_inf_mask((B, H, 1, cap), 0.1, seed * 8 + 5, dtype="f16").cuda()
    return q, kc, vc, torch.tensor(lens, dtype=torch.int32, device="cuda"), mask


def _close(a, b, la, lb):
    assert torch.equal(torch.isneginf(la), torch.isneginf(lb))
    fin = ~torch.isneginf(lb)
    assert (a.float() - b.float()).abs().max().item() <= 2e-2
    assert (a.float() - b.float()).abs().mean().item() <= 2e-3
    if fin.any():
        assert (la[fin] - lb[fin]).abs().max().item() <= 1e-2


def test_noalloc_matches_workspace_decode_twice():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    # first call: the decode configuration's shape (B=16, H=32, Hkv=8, cap=8192, D=128)
    lens1 = synth.kv_lengths(16, 8192, 4242).tolist()
    a1 = _inputs(16, 32, 8, 8192, 128, seed=4242, lens=lens1)
    # second call: other data and shorter sequences, so stale scratch from call 1 is present
    lens2 = [max(0, x // 3) for x in lens1]
    lens2[0] = 0
    a2 = _inputs(16, 32, 8, 8192, 128, seed=4343, lens=lens2)
    assert fa.decode_workspace_size(16, 32, 8, 8192, 128) <= fa.DECODE_STATIC_SCRATCH_BYTES
    for q, kc, vc, kl, m in (a1, a2):
        o_ref, l_ref = fa.decode(q, kc, vc, kl, SCALE, mask=m)
        o, l = fa.decode_noalloc(q, kc, vc, kl, SCALE, mask=m)
        torch.cuda.synchronize()
        _close(o, o_ref, l, l_ref)
    assert fa.device_status() == 0


def test_noalloc_refuses_oversized_workspace():
    import attention_flex_attn_b200 as fa
    lib = fa.load_library()
    B, H, Hkv, cap, D = 64, 64, 8, 65536, 128
    assert fa.decode_workspace_size(B, H, Hkv, cap, D) > fa.DECODE_STATIC_SCRATCH_BYTES
    p = torch.empty(16, dtype=torch.uint8, device="cuda")
    ptr = p.data_ptr()
    rc = lib.flex_attn_decode_noalloc(ptr, ptr, ptr, ptr, None, ptr, None, B, H, Hkv, cap, D, SCALE, 1, None)
    assert rc == 4  # FLEX_ERR_WORKSPACE, nothing launched
