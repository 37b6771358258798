"""CPU checks of the C ABI: the library loads, exports what the header declares, and
rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

import attention_flex_attn_b200 as fa
from attention_flex_attn_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def _declared():
    txt = open(os.path.join(ROOT, "include", "flex_attn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(flex_\w+)\s*\(", txt)))


def test_header_symbols_exported(lib):
    names = _declared()
    assert names, "no declarations found"
    assert sorted(fa.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        assert lib.flex_status_string(code)
    assert lib.flex_status_string(99) == b"unknown status"


def test_tile_sizes(lib):
    assert fa.tile_sizes(128) == (128, 128)
    assert fa.tile_sizes(64) == (128, 128)


def test_workspace_size(lib):
    # sized for the smallest split (128 positions): ceil(8192/128) = 64 splits;
    # o part [16*32, 64, 128] fp32 + lse part
    n = fa.decode_workspace_size(16, 32, 8, 8192, 128)
    assert n == 16 * 32 * 64 * 128 * 4 + 16 * 32 * 64 * 4
    assert fa.decode_workspace_size(0, 32, 8, 8192, 128) == 0


P = ctypes.c_void_p


def _fwd(lib, q=16, k=16, v=16, o=16, lse=None, B=1, H=2, Hkv=1, Sq=8, Skv=8, D=128, scale=0.1,
         score=0, mask=0, mp=None, dtype=0):
    return lib.flex_attn_fwd(P(q), P(k), P(v), P(o), P(lse), B, H, Hkv, Sq, Skv, D, scale, score, mask,
                             ctypes.byref(mp) if mp is not None else None, dtype, None)


def test_fwd_rejects_bad_args_on_host(lib):
    assert _fwd(lib, q=0) == 1
    assert _fwd(lib, B=0) == 1
    assert _fwd(lib, H=3, Hkv=2) == 1
    assert _fwd(lib, Sq=0) == 1
    assert _fwd(lib, scale=0.0) == 1
    assert _fwd(lib, scale=float("nan")) == 1
    assert _fwd(lib, D=96) == 2
    assert _fwd(lib, dtype=7) == 2
    assert _fwd(lib, score=5) == 1
    assert _fwd(lib, mask=9) == 1
    assert _fwd(lib, mask=2, mp=fa.ModParams(0, 0, 0, None)) == 1      # window < 1
    assert _fwd(lib, mp=fa.ModParams(1, 0, 1, None)) == 1              # tile map without buffer
    assert _fwd(lib, q=17) == 3
    assert _fwd(lib, lse=20) == 3
    st = fa.ModParams(0, 0, 0, None, None, None, None, 0, 18)         # status word not 4-byte aligned
    assert _fwd(lib, mp=st) == 3


def test_decode_rejects_bad_args_on_host(lib):
    def dec(q=16, k=16, v=16, kl=16, m=None, o=16, lse=None, B=2, H=4, Hkv=2, cap=64, D=128, scale=0.1,
            dtype=1, ws=16, wsb=1 << 20, split=0, status=None):
        dp = fa.DecodeParamsC(split, status)
        return lib.flex_attn_decode(P(q), P(k), P(v), P(kl), P(m), P(o), P(lse), B, H, Hkv, cap, D, scale,
                                    dtype, P(ws), wsb, ctypes.byref(dp), None)
    assert dec(kl=0) == 1
    assert dec(H=3) == 1
    assert dec(cap=0) == 1
    assert dec(D=80) == 2
    assert dec(ws=0) == 4
    assert dec(wsb=16) == 4
    assert dec(m=18) == 3
    assert dec(kl=4) == 3
    assert dec(split=64) == 1                 # split sizes are 128 and 256
    assert dec(split=512) == 1
    assert dec(status=6) == 3                 # status word not 4-byte aligned
    # a workspace that holds the 256-split partials only is enough for split 256
    small = 2 * 4 * 1 * 128 * 4 + 2 * 4 * 1 * 4  # B*H*ceil(64/256)*D*4 (a multiple of 256) + lse part
    assert dec(wsb=small - 1, split=256) == 4
    nalloc = lib.flex_attn_decode_noalloc
    dp = fa.DecodeParamsC(96, None)
    assert nalloc(P(16), P(16), P(16), P(16), None, P(16), None, 2, 4, 2, 64, 128, 0.1, 1, ctypes.byref(dp),
                  None) == 1


def test_mask_eval_rejects_bad_args(lib):
    assert lib.flex_attn_mask_eval(0, None, 0, 4, P(16), None) == 1
    assert lib.flex_attn_mask_eval(7, None, 4, 4, P(16), None) == 1
    assert lib.flex_attn_mask_eval(0, None, 4, 4, P(0), None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(fa.FlexAttnError):
        fa.fwd(q, q, q)


def test_static_scratch_limit_matches_header():
    txt = open(os.path.join(ROOT, "include", "flex_attn.h")).read()
    m = re.search(r"#define FLEX_DECODE_STATIC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", txt)
    assert m, "FLEX_DECODE_STATIC_SCRATCH_BYTES not found"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == fa.DECODE_STATIC_SCRATCH_BYTES


def test_selftest_rejects_bad_timeouts(lib):
    assert lib.flex_attn_selftest_wait_timeout(0, None) == 1
    assert lib.flex_attn_selftest_wait_timeout(2000001, None) == 1


def test_block_sparse_rejects_bad_args_on_host(lib):
    def bs(bm, Sq=8, Skv=8, **kw):
        return lib.flex_attn_fwd_block_sparse(P(16), P(16), P(16), P(16), None, 1, 2, 1, Sq, Skv, 128, 0.1, 0, 0,
                                              None, ctypes.byref(bm) if bm is not None else None, 0, None)

    def mask(num=32, idx=64, fnum=None, fidx=None, maxb=1, batch=1, heads=1, qb=128, kb=128):
        return fa.BlockMaskC(num, idx, fnum, fidx, maxb, batch, heads, qb, kb)
    assert bs(None) == 1
    assert bs(mask(num=None, idx=None)) == 1              # neither list
    assert bs(mask(idx=None)) == 1                        # counts without indices
    assert bs(mask(fnum=32)) == 1                         # full counts without indices
    assert bs(mask(maxb=0)) == 1
    assert bs(mask(batch=3)) == 1                         # batch must be 1 or B
    assert bs(mask(heads=3)) == 1                         # heads must be 1 or H
    assert bs(mask(qb=64)) == 2
    assert bs(mask(kb=256)) == 2
    assert bs(mask(), Skv=2048 * 128 + 1) == 2            # beyond what the bitmaps name
    assert bs(mask(num=34)) == 3                          # not 4-byte aligned
    assert bs(mask(fnum=32, fidx=66)) == 3


def test_captured_mods_rejected_on_host(lib):
    def fwd(score=0, mask=0, mp=None):
        return lib.flex_attn_fwd(P(16), P(16), P(16), P(16), None, 2, 2, 1, 8, 8, 128, 0.1, score, mask,
                                 ctypes.byref(mp) if mp is not None else None, 0, None)
    mp = lambda **kw: fa.ModParams(kw.get("window", 0), 0, 0, None, kw.get("slopes"), kw.get("oq"), kw.get("okv"),
                                   kw.get("n", 1))
    assert fwd(score=2) == 1                                  # slope table missing
    assert fwd(score=2, mp=mp(slopes=18)) == 3                # slope table misaligned
    assert fwd(score=3) == 1                                  # no such score_mod
    assert fwd(mask=5) == 1                                   # boundaries missing
    assert fwd(mask=6, mp=mp(oq=32, n=-1)) == 1               # negative document count
    assert fwd(mask=5, mp=mp(oq=34)) == 3                     # misaligned boundaries
    assert fwd(mask=6, mp=mp(oq=32, okv=66)) == 3
    assert fwd(mask=7) == 1                                   # no such mask_mod
    big = lib.flex_attn_fwd(P(16), P(16), P(16), P(16), None, 2, 2, 1, 8, 2048 * 128 + 1, 128, 0.1, 0, 5,
                            ctypes.byref(mp(oq=32)), 0, None)
    assert big == 2                                           # beyond the key-tile bitmaps
    assert lib.flex_attn_mask_eval(5, None, 4, 4, P(16), None) == 1


def test_bwd_rejects_bad_args_on_host(lib):
    def bwd(q=16, lse=32, ws=64, wsb=1 << 20, B=1, H=2, Hkv=1, Sq=8, Skv=8, D=128, scale=0.1, score=0, mask=0,
            mp=None, dtype=0):
        return lib.flex_attn_bwd(P(q), P(16), P(16), P(16), P(lse), P(16), P(16), P(16), P(16), B, H, Hkv, Sq, Skv, D,
                                 scale, score, mask, ctypes.byref(mp) if mp is not None else None, dtype, P(ws), wsb,
                                 None)
    assert bwd(q=0) == 1
    assert bwd(lse=0) == 1
    assert bwd(H=3, Hkv=2) == 1
    assert bwd(scale=-1.0) == 1
    assert bwd(D=96) == 2
    assert bwd(mask=9) == 1
    assert bwd(ws=0) == 4
    assert bwd(wsb=16) == 4
    assert bwd(q=24) == 3
    assert bwd(lse=34) == 3
    assert fa.bwd_workspace_size(2, 4, 300) == 2 * 2 * 4 * 384 * 4


def test_fwd_host_rejects_bad_args_on_host(lib):
    def fh(q=16, ws=64, wsb=1 << 30, D=128, H=2, Hkv=1, score=0, mask=0, mp=None):
        return lib.flex_attn_fwd_host(P(q), P(16), P(16), P(16), None, 1, H, Hkv, 8, 8, D, 0.1, score, mask,
                                      ctypes.byref(mp) if mp is not None else None, 0, P(ws), wsb, None)
    assert fh(q=0) == 1
    assert fh(H=3, Hkv=2) == 1
    assert fh(D=96) == 2
    assert fh(mask=9) == 1
    assert fh(score=7) == 1
    tile_map = fa.ModParams(0, 0, fa.FLAG_TILE_MAP, 16, None, None, None, 0, None)
    assert fh(mp=tile_map) == 1
    assert fh(ws=0) == 4
    assert fh(wsb=16) == 4
    assert fh(ws=24) == 3
    assert lib.flex_attn_fwd_host(P(16), P(16), P(16), P(16), None, 1, 2, 1, 8, 8, 128, -1.0, 0, 0, None, 0, P(64),
                                  1 << 30, None) == 1                       # scale <= 0
    assert fh(score=2) == 1                                                # slope table missing
    window0 = fa.ModParams(0, 0, 0, None, None, None, None, 0, None)
    assert fh(mask=2, mp=window0) == 1                                     # sliding window of 0
    # three chunk buffers (Q, K, V, O of hc kv heads, 256-byte aligned, and their LSE) and
    # the slope table: B=2 H=32 Hkv=32 S=8192 D=128 -> 16 chunks of 4 kv heads
    q_bytes = 4 * 8192 * 128 * 2
    lse_bytes = 4 * 8192 * 4
    assert fa.fwd_host_workspace_size(2, 32, 32, 8192, 8192, 128) == 3 * (4 * q_bytes + lse_bytes) + 256
    assert fa.fwd_host_workspace_size(2, 3, 2, 8, 8, 128) == 0
    # 16 or more batches: runs of whole batches, B=32 H=4 Hkv=2 S=100 D=64 -> runs of 2
    # batches (4 kv heads, 8 query heads) per chunk
    buf = 2 * (8 * 100 * 64 * 2) + 2 * (4 * 100 * 64 * 2) + 3328
    assert fa.fwd_host_workspace_size(32, 4, 2, 100, 100, 64) == 3 * buf + 256


def test_fp8_rejects_bad_args_on_host(lib):
    def f8(q=16, ws=64, wsb=1 << 24, D=128, scale=0.1, dq=1.0, dk=1.0, dv=1.0, score=0, mask=0, mp=None):
        return lib.flex_attn_fwd_fp8(P(q), P(16), P(16), P(16), None, 1, 2, 1, 8, 8, D, scale, dq, dk, dv, score,
                                     mask, ctypes.byref(mp) if mp is not None else None, P(ws), wsb, None)
    assert f8(q=0) == 1
    assert f8(D=96) == 2
    assert f8(dq=0.0) == 1
    assert f8(dv=float("inf")) == 1
    assert f8(mask=5) == 1                                   # document rules without boundaries
    assert f8(mp=fa.ModParams(0, 0, 1, None, None, None, None, 0)) == 1  # tile map flag without a buffer
    bm = fa.BlockMaskC(32, 64, None, None, 1, 3, 1, 128, 128)           # batch must be 1 or B
    assert lib.flex_attn_fwd_fp8_block_sparse(P(16), P(16), P(16), P(16), None, 1, 2, 1, 8, 8, 128, 0.1, 1.0, 1.0,
                                              1.0, 0, 0, None, ctypes.byref(bm), P(64), 1 << 24, None) == 1
    assert lib.flex_attn_fwd_fp8_block_sparse(P(16), P(16), P(16), P(16), None, 1, 2, 1, 8, 8, 128, 0.1, 1.0, 1.0,
                                              1.0, 0, 0, None, None, P(64), 1 << 24, None) == 1
    assert f8(ws=0) == 4
    assert f8(wsb=100) == 4
    assert f8(q=8) == 3
    assert fa.load_library().flex_attn_fwd_fp8_workspace_size(2, 4, 300, 128) == 2 * 4 * 128 * 384
    assert fa.load_library().flex_attn_fwd_fp8_workspace_size(2, 4, 300, 64) == 2 * 4 * 64 * 384
    assert fa.load_library().flex_attn_fwd_fp8_workspace_size(2, 4, 300, 96) == 0


def _declared_arity():
    """Parameter count of every function the header declares (void-parameter lists count 0)."""
    txt = open(os.path.join(ROOT, "include", "flex_attn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    txt = re.sub(r"//[^\n]*", "", txt)
    out = {}
    for m in re.finditer(r"\b(flex_\w+)\s*\(([^;{]*?)\)\s*;", txt):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_header(lib):
    """Every argtypes list the binding sets has exactly as many entries as the header's
    declaration has parameters, so a changed signature cannot be called with a stale one."""
    arity = _declared_arity()
    assert set(arity) == set(fa.EXPORTED)
    checked = 0
    for name, n in arity.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
        checked += 1
    assert checked >= len(arity) // 2


def _c_offsets():
    """offsetof/sizeof of the header's parameter structs, from a C compiler."""
    import subprocess
    import tempfile
    src = r"""
#include <stddef.h>
#include <stdio.h>
#include "flex_attn.h"
#define F(T, m) printf(#T "." #m " %zu\n", offsetof(T, m))
int main(void) {
  F(flex_mod_params_t, window); F(flex_mod_params_t, offset); F(flex_mod_params_t, flags);
  F(flex_mod_params_t, tile_map_out); F(flex_mod_params_t, alibi_slopes); F(flex_mod_params_t, doc_offsets_q);
  F(flex_mod_params_t, doc_offsets_kv); F(flex_mod_params_t, n_docs); F(flex_mod_params_t, status_out);
  F(flex_decode_params_t, split_size); F(flex_decode_params_t, status_out);
  F(flex_block_mask_t, kv_num_blocks); F(flex_block_mask_t, kv_indices); F(flex_block_mask_t, full_kv_num_blocks);
  F(flex_block_mask_t, full_kv_indices); F(flex_block_mask_t, max_blocks); F(flex_block_mask_t, batch);
  F(flex_block_mask_t, heads); F(flex_block_mask_t, q_block_size); F(flex_block_mask_t, kv_block_size);
  printf("sizeof.flex_mod_params_t %zu\nsizeof.flex_decode_params_t %zu\nsizeof.flex_block_mask_t %zu\n",
         sizeof(flex_mod_params_t), sizeof(flex_decode_params_t), sizeof(flex_block_mask_t));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "layout.c"), os.path.join(d, "layout")
        with open(c, "w") as f:
            f.write(src)
        subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), "-o", exe, c])
        out = subprocess.check_output([exe]).decode()
    return {k: int(v) for k, v in (line.split() for line in out.splitlines())}


def test_struct_layouts_match_header():
    """The binding's ctypes structures have the C layout of the header's structs (field
    offsets and sizes), so a field added on one side cannot shift the other's."""
    c = _c_offsets()
    for name, cls in (("flex_mod_params_t", fa.ModParams), ("flex_decode_params_t", fa.DecodeParamsC),
                      ("flex_block_mask_t", fa.BlockMaskC)):
        assert ctypes.sizeof(cls) == c[f"sizeof.{name}"], name
        for field, _ in cls._fields_:
            assert getattr(cls, field).offset == c[f"{name}.{field}"], (name, field)


def test_decode_shape_checks_on_cpu():
    """decode()/decode_noalloc() validate every tensor before anything launches: each
    mismatch below would otherwise make a kernel read or write past an allocation."""
    import torch
    B, H, Hkv, cap, D = 2, 4, 2, 64, 128
    f16 = torch.float16

    def args(**over):
        a = dict(q=torch.zeros(B, H, 1, D, dtype=f16), k_cache=torch.zeros(B, Hkv, cap, D, dtype=f16),
                 v_cache=torch.zeros(B, Hkv, cap, D, dtype=f16), kv_len=torch.zeros(B, dtype=torch.int32),
                 mask=torch.zeros(B, H, 1, cap, dtype=f16), out=torch.zeros(B, H, 1, D, dtype=f16),
                 lse_out=torch.zeros(B, H, 1, dtype=torch.float32))
        a.update(over)
        return a
    assert fa._check_decode_shapes(**args()) == (B, H, Hkv, cap, D)
    bad = [dict(kv_len=torch.zeros(B - 1, dtype=torch.int32)),              # short kv_len
           dict(kv_len=torch.zeros(B, dtype=torch.int64)),                  # wrong kv_len dtype
           dict(v_cache=torch.zeros(B, Hkv, cap // 2, D, dtype=f16)),       # smaller v_cache
           dict(v_cache=torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16)),
           dict(k_cache=torch.zeros(B + 1, Hkv, cap, D, dtype=f16)),        # batch mismatch
           dict(k_cache=torch.zeros(B, Hkv, cap, 64, dtype=f16)),           # head dim mismatch
           dict(mask=torch.zeros(B, H, 1, cap - 1, dtype=f16)),             # short mask
           dict(mask=torch.zeros(B, H, 1, cap, dtype=torch.float32)),       # fp32 mask
           dict(out=torch.zeros(B, H, 1, D // 2, dtype=f16)),               # small out
           dict(out=torch.zeros(B, H, 1, D, dtype=torch.bfloat16)),
           dict(lse_out=torch.zeros(B, H, dtype=torch.float32)),
           dict(lse_out=torch.zeros(B, H, 1, dtype=f16)),
           dict(q=torch.zeros(B, H, 2, D, dtype=f16)),                      # not one query row
           dict(q=torch.zeros(B, H, 1, D, dtype=torch.float32))]
    for over in bad:
        with pytest.raises(fa.FlexAttnError):
            fa._check_decode_shapes(**args(**over))


def test_fwd_shape_checks_on_cpu():
    import torch
    bf = torch.bfloat16
    q = torch.zeros(2, 4, 100, 64, dtype=bf)
    k = torch.zeros(2, 2, 80, 64, dtype=bf)
    assert fa._check_fwd_shapes(q, k, k) == (2, 4, 2, 100, 80, 64)
    with pytest.raises(fa.FlexAttnError):
        fa._check_fwd_shapes(q, k, torch.zeros(2, 2, 81, 64, dtype=bf))
    with pytest.raises(fa.FlexAttnError):
        fa._check_fwd_shapes(q, k, k, out=torch.zeros(2, 4, 99, 64, dtype=bf))
    with pytest.raises(fa.FlexAttnError):
        fa._check_fwd_shapes(q, k, k, out=torch.zeros(2, 4, 100, 64, dtype=torch.float16))
    with pytest.raises(fa.FlexAttnError):
        fa._check_fwd_shapes(q, k, k, lse_out=torch.zeros(2, 4, 100, dtype=bf))
    with pytest.raises(fa.FlexAttnError):
        fa._check_fwd_shapes(q, k, k, lse_out=torch.zeros(2, 4, 101, dtype=torch.float32))


def test_bwd_block_sparse_rejects_bad_args_on_host(lib):
    def bb(bm, ws=64, wsb=1 << 20, Skv=8):
        return lib.flex_attn_bwd_block_sparse(P(16), P(16), P(16), P(16), P(32), P(16), P(16), P(16), P(16), 1, 2, 1,
                                              8, Skv, 128, 0.1, 0, 0, None,
                                              ctypes.byref(bm) if bm is not None else None, 0, P(ws), wsb, None)

    def mask(num=32, idx=64, fnum=None, fidx=None, maxb=1, batch=1, heads=1, qb=128, kb=128):
        return fa.BlockMaskC(num, idx, fnum, fidx, maxb, batch, heads, qb, kb)
    assert bb(None) == 1
    assert bb(mask(num=None, idx=None)) == 1
    assert bb(mask(heads=3)) == 1
    assert bb(mask(qb=64)) == 2
    assert bb(mask(), Skv=2048 * 128 + 1) == 2
    assert bb(mask(num=34)) == 3
    assert bb(mask(), ws=0) == 4
    assert bb(mask(), wsb=100) == 4
    # statistics [2 * B * H * Sq_pad] floats, then per (b, kv head, key tile) 2 words per
    # ceil(G * n_qtiles / 32): B=2 H=4 Hkv=2 Sq=300 Skv=700 -> 3 query tiles, 6 key tiles
    assert lib.flex_attn_bwd_block_sparse_workspace_size(2, 4, 2, 300, 700) == 2 * 2 * 4 * 384 * 4 + 2 * 2 * 6 * 2 * 4
    assert lib.flex_attn_bwd_block_sparse_workspace_size(2, 3, 2, 300, 700) == 0
