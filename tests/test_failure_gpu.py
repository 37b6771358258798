"""Failure detection on the GPU without a fault: a bounded wait is made to run out (a
barrier nothing arrives on, 50 ms limit).  The kernel must end normally, report through
the device status word, and leave the context usable for real work."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def test_expired_wait_sets_status_and_context_survives():
    import attention_flex_attn_b200 as fa
    fa.load_library()
    fa.device_status(reset=True)
    t0 = time.perf_counter()
    fa.selftest_wait_timeout(50_000)
    st = fa.device_status(reset=True)   # synchronises
    dt = time.perf_counter() - t0
    assert st & 8, f"status {st:#x}: the self-test wait did not report its timeout"
    assert dt >= 0.045, f"the wait gave up after {dt * 1e3:.1f} ms, before its 50 ms limit"
    # the context still works: a forward right after matches the oracle
    q, k, v = synth.qkv(1, 2, 2, 130, 200, 64, seed=77)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), mask_mod="causal")
    torch.cuda.synchronize()
    ro, rl = oracle.fwd(q, k, v, mask_mod="causal")
    assert np.abs(o.float().cpu().numpy() - ro).max() < 2e-2
    assert np.abs(lse.cpu().numpy() - rl).max() < 1e-2
    assert fa.device_status() == 0
