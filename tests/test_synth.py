"""The seeded input generator: deterministic, counter based, the same stream on the CPU
(numpy) and through torch, and with the distributions the workloads name."""
import numpy as np
import torch

import synth


def test_deterministic_and_seed_dependent():
    a = synth.normal_tensor((3, 5, 7), 42)
    b = synth.normal_tensor((3, 5, 7), 42)
    c = synth.normal_tensor((3, 5, 7), 43)
    assert torch.equal(a, b) and not torch.equal(a, c)


def test_counter_based_prefix():
    """Element n does not depend on how many elements are drawn."""
    long = synth.normal_fp64(7, 1001)
    short = synth.normal_fp64(7, 10)
    np.testing.assert_array_equal(long[:10], short)


def test_torch_stream_matches_numpy():
    x = synth.normal_fp64(9, 4097)
    y = synth.normal_fp64_torch(9, 4097, "cpu").numpy()
    assert np.abs(x - y).max() < 1e-12
    a = synth.normal_tensor((64, 64), 9, dtype="bf16")
    b = synth.normal_tensor((64, 64), 9, dtype="bf16", device="cpu")
    assert (a.float() != b.float()).sum().item() <= 2  # last-ulp Box-Muller differences only


def test_moments_and_ranges():
    z = synth.normal_fp64(11, 200_000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    lens = synth.kv_lengths(10_000, 8192, 5)
    assert lens.min().item() >= 1 and lens.max().item() <= 8192
    assert abs(lens.double().mean().item() - 4096.5) < 100
    m = synth.bernoulli_neg_inf_mask((100_000,), 0.1, 3, dtype="f16")
    frac = torch.isneginf(m.float()).double().mean().item()
    assert abs(frac - 0.1) < 0.005 and torch.all((m == 0) | torch.isneginf(m.float()))
