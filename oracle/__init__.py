"""fp64 CPU oracle for flex attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / reference leg may import this package.  It shares no code
with the CUDA library: ``flex_oracle.c`` restates the method from its
definition (see the header of that file for the formulas and their sources).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
and ``tests/test_oracle_block_pins.py`` (closed forms, library special cases,
exact identities, hand-worked golden values); nothing is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flex_oracle.c")
_LIB = os.path.join(_HERE, "_flex_oracle.so")

SCORE_MODS = {"none": 0, "alibi": 1}
MASK_MODS = {"none": 0, "causal": 1, "sliding_window": 2, "kv_le_q_plus_offset": 3,
             # causal=True is the same keep rule as causal_via_mask
             "causal_fast": 1,
             # tensor-capturing: same document under per-batch boundary offsets (+ causal)
             "document": 5, "document_causal": 6}

_lib = None


def build(force: bool = False) -> str:
    """Compile flex_oracle.c into a shared library next to it (gcc -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.check_call(cmd)
    return _LIB


def _bind(lib):
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_fwd.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, I, I, I, P, P, P, I, P, I64, P, P, P, I]
    lib.oracle_fwd.restype = I
    lib.oracle_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, D, P, P, I]
    lib.oracle_decode.restype = I
    lib.oracle_mask_matrix.argtypes = [I, I, I, I, I, P, P, I, P]
    lib.oracle_mask_matrix.restype = I
    lib.oracle_tile_map.argtypes = [I, I, I, I, I, P, P, I, I, I, P]
    lib.oracle_tile_map.restype = I
    lib.oracle_alibi_slope.argtypes = [I, I]
    lib.oracle_alibi_slope.restype = D
    lib.oracle_e4m3_value.argtypes = [I]
    lib.oracle_e4m3_value.restype = D
    lib.oracle_fwd_block_sparse.argtypes = [P, P, P, I, I, I, I, I, I, I, D, I, I, I, I, P, P, P, I,
                                            P, P, P, P, I, I, I, P, I64, P, P, I]
    lib.oracle_fwd_block_sparse.restype = I
    lib.oracle_bwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, D, I, I, I, I, P, P, P, I, P, I64, P, P, P, I]
    lib.oracle_bwd.restype = I
    lib.oracle_bwd_block_sparse.argtypes = [P, P, P, P, I, I, I, I, I, I, I, D, I, I, I, I, P, P, P, I,
                                            P, P, P, P, I, I, I, P, I64, P, P, P, I]
    lib.oracle_bwd_block_sparse.restype = I
    return lib


def use_library(path=None):
    """Test hook: route the wrappers through another build of flex_oracle.c (for the
    mutation test of the pins); path None goes back to the normal build."""
    global _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        _lib = _bind(lib)
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return 0
    if t.dtype == torch.float16:
        return 1
    if t.dtype == torch.float8_e4m3fn:
        return 2
    raise TypeError(f"oracle takes bf16/f16/e4m3 tensors, got {t.dtype}")


def _bits(t: torch.Tensor) -> np.ndarray:
    """The raw bit patterns of a CPU bf16/f16 (16-bit) or e4m3 (8-bit) tensor (contiguous copy)."""
    if t.dtype == torch.float8_e4m3fn:
        return t.detach().cpu().contiguous().view(torch.uint8).numpy()
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _captured(B, H, mask_mod, alibi_slopes, doc_offsets, doc_offsets_kv):
    """float64 [H] slopes and int32 [B, n_docs + 1] boundary arrays (or None), and n_docs."""
    slopes = None
    if alibi_slopes is not None:
        if isinstance(alibi_slopes, torch.Tensor):
            alibi_slopes = alibi_slopes.detach().cpu().double().numpy()
        slopes = np.ascontiguousarray(np.asarray(alibi_slopes, dtype=np.float64).reshape(H))
    oq = okv = None
    n_docs = 0
    if mask_mod in ("document", "document_causal"):
        if doc_offsets is None:
            raise ValueError("document masks need doc_offsets")
        oq = _i32(doc_offsets).reshape(B, -1)
        okv = oq if doc_offsets_kv is None else _i32(doc_offsets_kv).reshape(B, -1)
        if okv.shape != oq.shape:
            raise ValueError("doc_offsets and doc_offsets_kv differ in shape")
        oq, okv = np.ascontiguousarray(oq), np.ascontiguousarray(okv)
        n_docs = oq.shape[1] - 1
    return slopes, oq, okv, n_docs


def _p(a):
    return None if a is None else a.ctypes.data


def fwd(q, k, v, scale=None, score_mod="none", mask_mod="none", window=0, offset=0,
        rows=None, want_probs=False, threads=None, alibi_slopes=None, doc_offsets=None,
        doc_offsets_kv=None):
    """Oracle forward.  q [B,H,Sq,D], k/v [B,Hkv,Skv,D] (CPU bf16/f16 tensors).

    rows: optional int64 array of flattened (b*H + h)*Sq + i row indices.
    alibi_slopes: [H] slopes for score_mod="alibi" (default: 2^(-8(h+1)/H)).
    doc_offsets / doc_offsets_kv: [B, n_docs + 1] document boundaries of the query / key
    positions for mask_mod "document" / "document_causal" (kv defaults to the query's).
    Returns (O, LSE[, P]) as float64 numpy arrays; O is [B,H,Sq,D] / LSE
    [B,H,Sq] for all rows, or [n,D] / [n] for a row subset.
    """
    lib = _load()
    B, H, Sq, D = q.shape
    slopes, oq, okv, n_docs = _captured(B, H, mask_mod, alibi_slopes, doc_offsets, doc_offsets_kv)
    Bk, Hkv, Skv, Dk = k.shape
    assert Bk == B and Dk == D and tuple(v.shape) == tuple(k.shape)
    assert q.dtype == k.dtype == v.dtype
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    if rows is None:
        n = B * H * Sq
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = int(rows_arr.size)
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    probs = np.zeros((n, Skv), dtype=np.float64) if want_probs else None
    rc = lib.oracle_fwd(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, _dtype_code(q),
                        B, H, Hkv, Sq, Skv, D, float(scale),
                        SCORE_MODS[score_mod], MASK_MODS[mask_mod], int(window), int(offset),
                        _p(slopes), _p(oq), _p(okv), n_docs,
                        None if rows_arr is None else rows_arr.ctypes.data, n,
                        o.ctypes.data, lse.ctypes.data,
                        None if probs is None else probs.ctypes.data,
                        int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_fwd rejected its arguments (rc={rc})")
    if rows is None:
        o = o.reshape(B, H, Sq, D)
        lse = lse.reshape(B, H, Sq)
        if probs is not None:
            probs = probs.reshape(B, H, Sq, Skv)
    return (o, lse, probs) if want_probs else (o, lse)


def bwd(q, k, v, dout, scale=None, score_mod="none", mask_mod="none", window=0, offset=0, groups=None,
        threads=None, alibi_slopes=None, doc_offsets=None, doc_offsets_kv=None):
    """Oracle backward: gradients dQ, dK, dV of sum(dout * O) for the forward with the same
    arguments.  groups: optional list of (b, hk) pairs (or flat b * Hkv + hk) to compute;
    None computes all.  Returns float64 arrays: dq [B,H,Sq,D], dk/dv [B,Hkv,Skv,D] for all
    groups, else dq [n, G, Sq, D] and dk/dv [n, Skv, D] in the order given."""
    lib = _load()
    B, H, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    assert tuple(dout.shape) == tuple(q.shape) and dout.dtype == q.dtype
    slopes, oq, okv, n_docs = _captured(B, H, mask_mod, alibi_slopes, doc_offsets, doc_offsets_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    G = H // Hkv
    if groups is None:
        g_arr, n = None, B * Hkv
    else:
        flat = [g[0] * Hkv + g[1] if isinstance(g, (tuple, list)) else int(g) for g in groups]
        g_arr = np.ascontiguousarray(np.asarray(flat, dtype=np.int64))
        n = int(g_arr.size)
    dq = np.zeros((n, G, Sq, D))
    dk = np.zeros((n, Skv, D))
    dv = np.zeros((n, Skv, D))
    qb, kb, vb, ob = _bits(q), _bits(k), _bits(v), _bits(dout)
    rc = lib.oracle_bwd(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, ob.ctypes.data, _dtype_code(q),
                        B, H, Hkv, Sq, Skv, D, float(scale), SCORE_MODS[score_mod], MASK_MODS[mask_mod],
                        int(window), int(offset), _p(slopes), _p(oq), _p(okv), n_docs,
                        None if g_arr is None else g_arr.ctypes.data, n,
                        dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_bwd rejected its arguments (rc={rc})")
    if groups is None:
        return dq.reshape(B, H, Sq, D), dk.reshape(B, Hkv, Skv, D), dv.reshape(B, Hkv, Skv, D)
    return dq, dk, dv


def _block_arrays(kv_num, kv_idx, full_num, full_idx, B, H, nq):
    """The lists broadcast to [B, H, nq(, max_blocks)] int32 (either pair may be None)."""
    kn, ki, fn, fi = _i32(kv_num), _i32(kv_idx), _i32(full_num), _i32(full_idx)
    if kn is None and fn is None:
        raise ValueError("a block mask needs at least one of the partial / full lists")
    max_blocks = (ki if ki is not None else fi).shape[-1]

    def expand(a, tail):
        return None if a is None else np.ascontiguousarray(np.broadcast_to(a, (B, H, nq) + tail))
    return expand(kn, ()), expand(ki, (max_blocks,)), expand(fn, ()), expand(fi, (max_blocks,)), max_blocks


def bwd_block_sparse(q, k, v, dout, kv_num, kv_idx, full_num=None, full_idx=None, scale=None,
                     score_mod="none", mask_mod="none", window=0, offset=0, bm=128, bn=128, groups=None,
                     threads=None, alibi_slopes=None, doc_offsets=None, doc_offsets_kv=None):
    """Oracle backward of the block-sparse forward: bwd() with the keep rule of
    fwd_block_sparse() (lists as there).  Returns (dq, dk, dv) like bwd()."""
    lib = _load()
    B, H, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    assert tuple(dout.shape) == tuple(q.shape) and dout.dtype == q.dtype
    slopes, oq, okv, n_docs = _captured(B, H, mask_mod, alibi_slopes, doc_offsets, doc_offsets_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    kn, ki, fn, fi, max_blocks = _block_arrays(kv_num, kv_idx, full_num, full_idx, B, H, -(-Sq // bm))
    G = H // Hkv
    if groups is None:
        g_arr, n = None, B * Hkv
    else:
        flat = [g[0] * Hkv + g[1] if isinstance(g, (tuple, list)) else int(g) for g in groups]
        g_arr = np.ascontiguousarray(np.asarray(flat, dtype=np.int64))
        n = int(g_arr.size)
    dq = np.zeros((n, G, Sq, D))
    dk = np.zeros((n, Skv, D))
    dv = np.zeros((n, Skv, D))
    qb, kb, vb, ob = _bits(q), _bits(k), _bits(v), _bits(dout)
    rc = lib.oracle_bwd_block_sparse(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, ob.ctypes.data, _dtype_code(q),
                                     B, H, Hkv, Sq, Skv, D, float(scale), SCORE_MODS[score_mod], MASK_MODS[mask_mod],
                                     int(window), int(offset), _p(slopes), _p(oq), _p(okv), n_docs,
                                     _p(kn), _p(ki), _p(fn), _p(fi), int(max_blocks), int(bm), int(bn),
                                     None if g_arr is None else g_arr.ctypes.data, n,
                                     dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_bwd_block_sparse rejected its arguments (rc={rc})")
    if groups is None:
        return dq.reshape(B, H, Sq, D), dk.reshape(B, Hkv, Skv, D), dv.reshape(B, Hkv, Skv, D)
    return dq, dk, dv


def e4m3_value(bits: int) -> float:
    """The exact value of an 8-bit e4m3 (E4M3FN) code."""
    return float(_load().oracle_e4m3_value(int(bits)))


def fwd_fp8(q8, k8, v8, descale_q=1.0, descale_k=1.0, descale_v=1.0, scale=None, **kw):
    """Oracle forward on e4m3 inputs with per-tensor descales: q = descale_q * q8 (and so
    on) exactly; returns (O, LSE) of the plain definition on those values (P unrounded)."""
    D = q8.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o, lse = fwd(q8, k8, v8, scale=float(scale) * float(descale_q) * float(descale_k), **kw)
    return o * float(descale_v), lse


def _i32(a):
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def fwd_block_sparse(q, k, v, kv_num, kv_idx, full_num=None, full_idx=None, scale=None,
                     score_mod="none", mask_mod="none", window=0, offset=0, bm=128, bn=128,
                     rows=None, threads=None, alibi_slopes=None, doc_offsets=None, doc_offsets_kv=None):
    """Oracle forward with a block mask (BlockMask: FlyDSL PR 931 "Add flex_attention
    (score_mod / mask_mod) ...", Out of scope, names block sparsity as the next phase;
    the list convention is PyTorch's).

    kv_num / full_num: [Bm, Hm, ceil(Sq/bm)] int32 block counts; kv_idx / full_idx:
    [Bm, Hm, ceil(Sq/bm), max_blocks] int32 key-block indices; Bm in {1, B} and Hm in
    {1, H} broadcast like numpy.  Either pair may be None (no blocks of that kind).
    Key j of query row i is kept iff j < Skv and its block j // bn is listed as full
    for the tile i // bm, or listed as partial and mask_mod(i, j) holds.  A count is
    clamped to [0, max_blocks]; an index outside [0, ceil(Skv/bn)) names no block.
    Returns (O, LSE) like fwd()."""
    lib = _load()
    B, H, Sq, D = q.shape
    _, Hkv, Skv, _ = k.shape
    slopes, oq, okv, n_docs = _captured(B, H, mask_mod, alibi_slopes, doc_offsets, doc_offsets_kv)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    nq = -(-Sq // bm)
    kn, ki, fn, fi = _i32(kv_num), _i32(kv_idx), _i32(full_num), _i32(full_idx)
    if kn is None and fn is None:
        raise ValueError("a block mask needs at least one of the partial / full lists")
    max_blocks = (ki if ki is not None else fi).shape[-1]

    def expand(a, tail):
        return None if a is None else np.ascontiguousarray(np.broadcast_to(a, (B, H, nq) + tail))
    kn, fn = expand(kn, ()), expand(fn, ())
    ki, fi = expand(ki, (max_blocks,)), expand(fi, (max_blocks,))
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    if rows is None:
        n, rows_arr = B * H * Sq, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = int(rows_arr.size)
    o = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = lib.oracle_fwd_block_sparse(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, _dtype_code(q),
                                     B, H, Hkv, Sq, Skv, D, float(scale), SCORE_MODS[score_mod],
                                     MASK_MODS[mask_mod], int(window), int(offset),
                                     _p(slopes), _p(oq), _p(okv), n_docs,
                                     ptr(kn), ptr(ki), ptr(fn), ptr(fi), int(max_blocks), int(bm), int(bn),
                                     None if rows_arr is None else rows_arr.ctypes.data, n,
                                     o.ctypes.data, lse.ctypes.data, int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_fwd_block_sparse rejected its arguments (rc={rc})")
    if rows is None:
        return o.reshape(B, H, Sq, D), lse.reshape(B, H, Sq)
    return o, lse


def block_mask_from_tile_map(tmap, B, H, max_blocks=None):
    """Partial/full block lists that reproduce a tile map (2 -> partial, 1 -> full)."""
    nq, nk = tmap.shape
    mb = max_blocks or nk
    kv_num = np.zeros((B, H, nq), np.int32)
    kv_idx = np.zeros((B, H, nq, mb), np.int32)
    full_num = np.zeros((B, H, nq), np.int32)
    full_idx = np.zeros((B, H, nq, mb), np.int32)
    for t in range(nq):
        part = [u for u in range(nk) if tmap[t, u] == 2]
        full = [u for u in range(nk) if tmap[t, u] == 1]
        kv_num[:, :, t] = len(part)
        kv_idx[:, :, t, :len(part)] = part
        full_num[:, :, t] = len(full)
        full_idx[:, :, t, :len(full)] = full
    return kv_num, kv_idx, full_num, full_idx


def decode(q, k_cache, v_cache, kv_len, scale, mask=None, threads=None):
    """Oracle decode.  q [B,H,1,D]; caches [B,Hkv,cap,D]; kv_len [B] int32;
    mask optional [B,H,1,cap] (f16/bf16).  Returns (O [B,H,1,D], LSE [B,H,1])."""
    lib = _load()
    B, H, one, D = q.shape
    assert one == 1
    _, Hkv, cap, _ = k_cache.shape
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    lens = np.ascontiguousarray(kv_len.detach().cpu().numpy().astype(np.int32))
    mb = _bits(mask) if mask is not None else None
    mdt = _dtype_code(mask) if mask is not None else 0
    o = np.zeros((B * H, D), dtype=np.float64)
    lse = np.zeros((B * H,), dtype=np.float64)
    rc = lib.oracle_decode(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, lens.ctypes.data,
                           None if mb is None else mb.ctypes.data, mdt, _dtype_code(q),
                           B, H, Hkv, cap, D, float(scale), o.ctypes.data, lse.ctypes.data,
                           int(threads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_decode rejected its arguments (rc={rc})")
    return o.reshape(B, H, 1, D), lse.reshape(B, H, 1)


def mask_matrix(mask_mod, Sq, Skv, window=0, offset=0, doc_offsets=None, doc_offsets_kv=None) -> np.ndarray:
    """uint8 [Sq, Skv]: 1 where mask_mod keeps (i, j) (document masks: one batch's
    boundaries, [n_docs + 1])."""
    lib = _load()
    _, oq, okv, n_docs = _captured(1, 1, mask_mod, None, doc_offsets, doc_offsets_kv)
    out = np.zeros((Sq, Skv), dtype=np.uint8)
    rc = lib.oracle_mask_matrix(MASK_MODS[mask_mod], Sq, Skv, int(window), int(offset), _p(oq), _p(okv), n_docs,
                                out.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_mask_matrix rejected its arguments (rc={rc})")
    return out


def tile_map(mask_mod, Sq, Skv, window=0, offset=0, bm=128, bn=128, doc_offsets=None,
             doc_offsets_kv=None) -> np.ndarray:
    """uint8 [ceil(Sq/bm), ceil(Skv/bn)]: 0 EMPTY, 1 FULL, 2 PARTIAL."""
    lib = _load()
    _, oq, okv, n_docs = _captured(1, 1, mask_mod, None, doc_offsets, doc_offsets_kv)
    nq, nk = -(-Sq // bm), -(-Skv // bn)
    out = np.zeros((nq, nk), dtype=np.uint8)
    rc = lib.oracle_tile_map(MASK_MODS[mask_mod], Sq, Skv, int(window), int(offset), _p(oq), _p(okv), n_docs,
                             bm, bn, out.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_tile_map rejected its arguments (rc={rc})")
    return out


def alibi_slope(h: int, H: int) -> float:
    return float(_load().oracle_alibi_slope(h, H))


def fwd_flops(B, H, Sq, Skv, D) -> float:
    """Dense forward work 4*B*H*Sq*Skv*D (two matmuls of 2*Sq*Skv*D each)."""
    return 4.0 * B * H * Sq * Skv * D
