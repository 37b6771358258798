"""GPU parity of flex_attn_fwd_host (the forward on host buffers, copies pipelined with
the kernels by chunks of kv heads) against the fp64 oracle and against flex_attn_fwd on
the same values.

The operation is the forward of FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod)
on the generic flash-attention kernel" (Summary); only where the operands live differs.
Each chunk runs the same kernels on a contiguous range of (batch, kv head) pairs, so its
rows equal flex_attn_fwd's up to the summation order of a split last round of units
(that split depends on the number of units per launch); with the built-in alibi the
chunks read a slope table the library fills with the kernels' own formula, and document
masks read their batch's boundaries.
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


def _pinned(*ts):
    return [t.cpu().contiguous().pin_memory() for t in ts]


MODS = [
    dict(),
    dict(mask_mod="causal", score_mod="alibi"),
    dict(mask_mod="sliding_window", window=200),
    dict(score_mod="alibi", alibi_slopes=np.array([0.3, -0.1, 0.05, 0.0, 0.5, 0.25, -0.2, 0.125], np.float32)),
    dict(mask_mod="document_causal", doc_offsets=np.array([[0, 300, 301, 800, 1000], [0, 50, 600, 900, 1000]],
                                                          np.int32)),
]


@pytest.mark.parametrize("mods", MODS, ids=["no_mod", "causal_alibi", "window", "slopes", "documents"])
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "f16")])
def test_gqa_against_oracle_and_device_forward(mods, D, dtype):
    """B2 H8 Hkv2 (four chunks of one kv head), Sq = Skv = 1000 (ragged tiles)."""
    fa = _fa()
    B, H, Hkv, S = 2, 8, 2, 1000
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=120 + D, dtype=dtype)
    m = dict(mods)
    for key in ("alibi_slopes", "doc_offsets"):
        if m.get(key) is not None:
            m[key] = torch.as_tensor(m[key]).cuda()
    hq, hk, hv = _pinned(q, k, v)
    o, lse = fa.fwd_host(hq, hk, hv, **m)
    od, ld = fa.fwd(q.cuda(), k.cuda(), v.cuda(), **m)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    assert o.device.type == "cpu" and lse.device.type == "cpu"
    assert (o.float() - od.cpu().float()).abs().max().item() <= 4e-3
    fin = torch.isfinite(ld.cpu())
    assert torch.equal(torch.isfinite(lse), fin)
    assert (lse[fin] - ld.cpu()[fin]).abs().max().item() <= 1e-5
    ro, rl = oracle.fwd(q, k, v, scale=1.0 / math.sqrt(D), **mods)
    compare(o, lse, ro, rl, f"fwd_host {mods}")


def test_bench_size_equals_device_forward_bitwise():
    """The bench's workload, B2 H32 S8192 D128 bf16 no_mod, from pinned host memory: every
    chunk runs the per-unit kernel over whole units, as the device call does, so the
    results are bit-identical; sampled rows against the oracle."""
    fa = _fa()
    B, H, S, D = 2, 32, 8192, 128
    q, k, v = synth.qkv(B, H, H, S, S, D, seed=4000, sigma=0.5, device="cuda")
    hq, hk, hv = _pinned(q, k, v)
    o, lse = fa.fwd_host(hq, hk, hv)
    od, ld = fa.fwd(q, k, v)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    assert torch.equal(o, od.cpu()) and torch.equal(lse, ld.cpu())
    rows = sample_rows(B, H, S, 512, 121, must=[(0, 0, 0), (1, 31, 8191), (0, 16, 4096)])
    ro, rl = oracle.fwd(hq, hk, hv, scale=1.0 / math.sqrt(D), rows=rows)
    compare(gather_rows(o, rows), gather_rows(lse, rows), ro, rl, "fwd_host bench size")


def test_without_lse_and_into_given_buffers():
    fa = _fa()
    B, H, Hkv, S, D = 1, 4, 4, 300, 128
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=122)
    hq, hk, hv = _pinned(q, k, v)
    out = torch.full(q.shape, float("nan"), dtype=q.dtype).pin_memory()
    ws = torch.empty(fa.fwd_host_workspace_size(B, H, Hkv, S, S, D), dtype=torch.uint8, device="cuda")
    o, lse = fa.fwd_host(hq, hk, hv, mask_mod="causal", return_lse=False, out=out, workspace=ws)
    assert lse is None and o is out
    od, _ = fa.fwd(q.cuda(), k.cuda(), v.cuda(), mask_mod="causal")
    assert (o.float() - od.cpu().float()).abs().max().item() <= 4e-3
    o2, _ = fa.fwd_host(hq, hk, hv, mask_mod="causal", return_lse=False, workspace=ws)  # workspace reused
    assert torch.equal(o2, o)


def test_many_batches_run_in_batch_chunks():
    """B = 40 (at least 16 batches: chunks are runs of whole batches), GQA 4/2, ragged
    Sq = Skv = 200, D = 64 f16, causal documents with per-batch boundaries and the built-in
    alibi: against the oracle (all rows) and the device forward."""
    fa = _fa()
    B, H, Hkv, S, D = 40, 4, 2, 200, 64
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=123, dtype="f16")
    rng = np.random.default_rng(124)
    offs = np.array([[0, *sorted(rng.integers(1, S, size=2).tolist()), S] for _ in range(B)], np.int32)
    mods = dict(mask_mod="document_causal", doc_offsets=offs, score_mod="alibi")
    m = dict(mods, doc_offsets=torch.as_tensor(offs).cuda())
    hq, hk, hv = _pinned(q, k, v)
    o, lse = fa.fwd_host(hq, hk, hv, **m)
    od, ld = fa.fwd(q.cuda(), k.cuda(), v.cuda(), **m)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    assert (o.float() - od.cpu().float()).abs().max().item() <= 4e-3
    ro, rl = oracle.fwd(q, k, v, scale=1.0 / math.sqrt(D), **mods)
    compare(o, lse, ro, rl, "fwd_host batch runs")


def test_pageable_host_memory():
    """Pageable (not pinned) host tensors: the copies serialise but the results are those
    of the pinned case, bit for bit."""
    fa = _fa()
    B, H, Hkv, S, D = 1, 8, 2, 700, 128
    q, k, v = synth.qkv(B, H, Hkv, S, S, D, seed=125)
    op, lp = fa.fwd_host(*_pinned(q, k, v), mask_mod="sliding_window", window=300)
    oq, lq = fa.fwd_host(q.contiguous(), k.contiguous(), v.contiguous(), mask_mod="sliding_window", window=300,
                         out=torch.empty(q.shape, dtype=q.dtype), lse_out=torch.empty((B, H, S)))
    assert not oq.is_pinned()
    assert torch.equal(op, oq) and torch.equal(lp, lq)
