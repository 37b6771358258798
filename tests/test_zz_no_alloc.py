"""flex_attn_decode_noalloc: the decode entry point for callers that cannot allocate.

Hosts that pass only inputs and outputs, processes whose device memory budget is
already reserved, and decode loops that cannot afford the device-wide synchronisation
of cudaMalloc/cudaFree call this variant; its scratch lives in an array compiled into
the library.  These tests call it through the C ABI twice in a row (with different
inputs, so the second call runs over the first call's leftover scratch) and check each
result against flex_attn_decode with a caller-allocated workspace, within the parity
tolerances of the other decode tests, and rows of it against the fp64 oracle.  The
cases cover both decode kernels (one query head per kv head, Hkv = 32; grouped heads,
Hkv = 8), f16 and bf16, D = 128 and 64, and both split sizes.  A size whose workspace
exceeds the compiled-in limit is refused.  Kept in a file of its own so that pytest
collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

SCALE = 0.08837890625


def _inputs(B, H, Hkv, cap, D, seed, lens, dtype="f16"):
    q = synth.normal_tensor((B, H, 1, D), seed * 8 + 1, dtype=dtype, device="cuda")
    kc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 2, dtype=dtype, device="cuda")
    vc = synth.normal_tensor((B, Hkv, cap, D), seed * 8 + 3, dtype=dtype, device="cuda")
    mask = synth.bernoulli_neg_inf_mask((B, H, 1, cap), 0.1, seed * 8 + 5, dtype=dtype).cuda()
    return q, kc, vc, torch.tensor(lens, dtype=torch.int32, device="cuda"), mask


def _close(a, b, la, lb):
    assert torch.equal(torch.isneginf(la), torch.isneginf(lb))
    fin = ~torch.isneginf(lb)
    assert (a.float() - b.float()).abs().max().item() <= 2e-2
    assert (a.float() - b.float()).abs().mean().item() <= 2e-3
    if fin.any():
        assert (la[fin] - lb[fin]).abs().max().item() <= 1e-2


def _oracle_rows(args, o, l, batches):
    """Rows of batches `batches` (all heads) against the oracle: O max-abs 2e-2, mean-abs
    2e-3, LSE 1e-2; rows without keys exactly O = +0, LSE = -inf."""
    q, kc, vc, kl, m = args
    sel = torch.tensor(batches)
    ro, rl = oracle.decode(q.cpu()[sel], kc.cpu()[sel], vc.cpu()[sel], kl.cpu()[sel], SCALE, mask=m.cpu()[sel])
    go = o.cpu()[sel].float().numpy().astype(np.float64)
    gl = l.cpu()[sel].numpy().astype(np.float64)
    ro, rl = np.asarray(ro).reshape(go.shape), np.asarray(rl).reshape(gl.shape)
    dead = np.isneginf(rl)
    assert np.array_equal(np.isneginf(gl), dead)
    assert np.all(go[dead] == 0.0) and not np.any(np.signbit(go[dead]))
    err = np.abs(go - ro)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    if (~dead).any():
        assert np.abs(gl[~dead] - rl[~dead]).max() <= 1e-2


@pytest.mark.parametrize("Hkv,D,dtype,split", [(8, 128, "f16", 0), (32, 128, "f16", 0), (8, 64, "bf16", 0),
                                               (32, 64, "bf16", 128)])
def test_noalloc_matches_workspace_decode_twice(Hkv, D, dtype, split):
    import attention_flex_attn_b200 as fa
    fa.load_library()
    B, H, cap = 16, 32, 8192
    # first call: the decode configuration's shape (B=16, H=32, cap=8192)
    lens1 = synth.kv_lengths(B, cap, 4242).tolist()
    a1 = _inputs(B, H, Hkv, cap, D, seed=4242 + Hkv + D, lens=lens1, dtype=dtype)
    # second call: other data and shorter sequences, so stale scratch from call 1 is present
    lens2 = [max(0, x // 3) for x in lens1]
    lens2[0] = 0
    a2 = _inputs(B, H, Hkv, cap, D, seed=4343 + Hkv + D, lens=lens2, dtype=dtype)
    for i, (q, kc, vc, kl, m) in enumerate((a1, a2)):
        o_ref, l_ref = fa.decode(q, kc, vc, kl, SCALE, mask=m, split_size=split)
        o, l = fa.decode_noalloc(q, kc, vc, kl, SCALE, mask=m, split_size=split)
        torch.cuda.synchronize()
        _close(o, o_ref, l, l_ref)
        if i == 1:
            _oracle_rows((q, kc, vc, kl, m), o, l, [0, 1, 7])
    assert fa.device_status() == 0


def test_noalloc_refuses_oversized_workspace():
    import attention_flex_attn_b200 as fa
    lib = fa.load_library()
    B, H, Hkv, cap, D = 64, 64, 8, 65536, 128
    assert fa.decode_workspace_size(B, H, Hkv, cap, D) > fa.DECODE_STATIC_SCRATCH_BYTES
    p = torch.empty(16, dtype=torch.uint8, device="cuda")
    ptr = p.data_ptr()
    rc = lib.flex_attn_decode_noalloc(ptr, ptr, ptr, ptr, None, ptr, None, B, H, Hkv, cap, D, SCALE, 1, None, None)
    assert rc == 4  # FLEX_ERR_WORKSPACE, nothing launched
    # the decode configuration fits at 256-position splits but not at 128
    dp = fa.DecodeParamsC(128, None)
    rc = lib.flex_attn_decode_noalloc(ptr, ptr, ptr, ptr, None, ptr, None, 16, 32, 8, 8192, 128, SCALE, 1,
                                      ctypes.byref(dp), None)
    assert rc == 4
