"""Shared helpers for the parity tests: tolerances and comparisons.

Tolerances (bf16/f16 outputs vs the fp64 oracle): O max-abs 2e-2, O mean-abs 2e-3,
LSE abs 1e-2 on finite rows; rows the oracle reports fully masked must come back as
LSE == -inf and O == +0 exactly; no NaN anywhere.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-2


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """o_gpu/lse_gpu: torch (any device) already selected to the same rows as o_ref/lse_ref."""
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    l = lse_gpu.detach().float().cpu().numpy().astype(np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64).reshape(o.shape)
    lse_ref = np.asarray(lse_ref, dtype=np.float64).reshape(l.shape)
    assert not np.isnan(o).any(), f"{what}: NaN in O"
    assert not np.isnan(l).any(), f"{what}: NaN in LSE"
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l), dead), f"{what}: fully-masked rows differ"
    if dead.any():
        od = o[dead]
        assert np.all(od == 0.0) and not np.any(np.signbit(od)), f"{what}: masked rows not +0"
    err = np.abs(o - o_ref)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    assert max_abs <= O_MAX_ABS, f"{what}: O max-abs {max_abs:.3e}"
    assert mean_abs <= O_MEAN_ABS, f"{what}: O mean-abs {mean_abs:.3e}"
    if (~dead).any():
        lerr = float(np.abs(l[~dead] - lse_ref[~dead]).max())
        assert lerr <= LSE_ABS, f"{what}: LSE abs {lerr:.3e}"
    return max_abs, mean_abs


def sample_rows(B, H, Sq, n, seed, must=()):
    """Sorted unique flattened row ids (b*H + h)*Sq + i: n random + the given (b,h,i) rows."""
    rng = np.random.default_rng(seed)
    total = B * H * Sq
    pick = set(rng.choice(total, size=min(n, total), replace=False).tolist())
    for b, h, i in must:
        if i < Sq:
            pick.add((b * H + h) * Sq + i)
    return np.array(sorted(pick), dtype=np.int64)


def gather_rows(t, rows):
    """t [B,H,S,...] -> rows of the flattened [B*H*S, ...] view."""
    flat = t.reshape(-1, *t.shape[3:]) if t.dim() > 3 else t.reshape(-1)
    return flat[torch.as_tensor(rows, device=t.device)]


def random_block_lists(rng, B, H, nq, nk, max_blocks, p_full=0.3, p_part=0.3):
    """Random block-mask lists (numpy int32): counts [B,H,nq], indices [B,H,nq,max_blocks]
    for partial and full blocks, with the irregularities a caller may pass -- a repeated
    index, an index naming no block (-1, nk, nk+5), garbage after the count, counts above
    max_blocks or below 0."""
    kn = np.zeros((B, H, nq), np.int32)
    ki = np.zeros((B, H, nq, max_blocks), np.int32)
    fn = np.zeros((B, H, nq), np.int32)
    fi = np.zeros((B, H, nq, max_blocks), np.int32)
    for b in range(B):
        for h in range(H):
            for t in range(nq):
                for num, idx, pr in ((kn, ki, p_part), (fn, fi, p_full)):
                    chosen = [u for u in range(nk) if rng.random() < pr]
                    if chosen and rng.random() < 0.3:
                        chosen.append(chosen[0])            # a duplicate
                    if rng.random() < 0.2:
                        chosen.append(int(rng.choice([-1, nk, nk + 5])))  # names no block
                    rng.shuffle(chosen)
                    chosen = chosen[:max_blocks]
                    idx[b, h, t, :len(chosen)] = chosen
                    idx[b, h, t, len(chosen):] = rng.integers(-3, nk + 3, max_blocks - len(chosen))
                    c = len(chosen)
                    r = rng.random()
                    num[b, h, t] = c if r < 0.8 else (max_blocks + 3 if r < 0.9 else -2)
    return kn, ki, fn, fi
