"""Python binding for the sm_100a flex-attention library (libflexattn.so).

Argument marshalling only: every step of the computation runs in the CUDA kernels
behind the C ABI of ``include/flex_attn.h``.  Tensors are torch CUDA tensors; the
binding passes their device pointers and the current CUDA stream.  There is no
fallback: if the shared library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflexattn.so")

# enum values of include/flex_attn.h
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "misaligned", 4: "workspace",
          5: "CUDA error", 6: "device timeout"}
DTYPES = {torch.bfloat16: 0, torch.float16: 1}
SCORE_MODS = {"none": 0, "alibi": 1}
SCORE_ALIBI_SLOPES = 2  # alibi with a captured slope tensor
MASK_MODS = {"none": 0, "causal": 1, "sliding_window": 2, "kv_le_q_plus_offset": 3, "causal_fast": 4,
             "document": 5, "document_causal": 6}
FLAG_TILE_MAP = 1

# The symbols include/flex_attn.h declares.
EXPORTED = ["flex_attn_fwd", "flex_attn_fwd_block_sparse", "flex_attn_fwd_host_workspace_size", "flex_attn_fwd_host",
            "flex_attn_fwd_fp8_workspace_size", "flex_attn_fwd_fp8",
            "flex_attn_fwd_fp8_block_sparse",
            "flex_attn_bwd_workspace_size", "flex_attn_bwd",
            "flex_attn_bwd_block_sparse_workspace_size", "flex_attn_bwd_block_sparse",
            "flex_attn_decode_workspace_size", "flex_attn_decode",
            "flex_attn_decode_noalloc", "flex_attn_mask_eval", "flex_attn_selftest_wait_timeout",
            "flex_attn_tile_sizes", "flex_attn_device_status", "flex_status_string"]


class FlexAttnError(RuntimeError):
    pass


class ModParams(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int32), ("offset", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("tile_map_out", ctypes.c_void_p),
                ("alibi_slopes", ctypes.c_void_p), ("doc_offsets_q", ctypes.c_void_p),
                ("doc_offsets_kv", ctypes.c_void_p), ("n_docs", ctypes.c_int32),
                ("status_out", ctypes.c_void_p)]


class DecodeParamsC(ctypes.Structure):
    """flex_decode_params_t of include/flex_attn.h."""
    _fields_ = [("split_size", ctypes.c_int32), ("status_out", ctypes.c_void_p)]


class BlockMaskC(ctypes.Structure):
    """flex_block_mask_t of include/flex_attn.h."""
    _fields_ = [("kv_num_blocks", ctypes.c_void_p), ("kv_indices", ctypes.c_void_p),
                ("full_kv_num_blocks", ctypes.c_void_p), ("full_kv_indices", ctypes.c_void_p),
                ("max_blocks", ctypes.c_int32), ("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("q_block_size", ctypes.c_int32), ("kv_block_size", ctypes.c_int32)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libflexattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FlexAttnError(f"{path} is missing: run `python -m attention_flex_attn_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.flex_attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, ctypes.POINTER(ModParams), I, P]
    lib.flex_attn_fwd.restype = I
    lib.flex_attn_fwd_block_sparse.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, ctypes.POINTER(ModParams),
                                               ctypes.POINTER(BlockMaskC), I, P]
    lib.flex_attn_fwd_block_sparse.restype = I
    lib.flex_attn_fwd_host_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.flex_attn_fwd_host_workspace_size.restype = SZ
    lib.flex_attn_fwd_host.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, ctypes.POINTER(ModParams), I, P,
                                       SZ, P]
    lib.flex_attn_fwd_host.restype = I
    lib.flex_attn_fwd_fp8_workspace_size.argtypes = [I, I, I, I]
    lib.flex_attn_fwd_fp8_workspace_size.restype = SZ
    lib.flex_attn_fwd_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, F, F, F, I, I, ctypes.POINTER(ModParams),
                                      P, SZ, P]
    lib.flex_attn_fwd_fp8.restype = I
    lib.flex_attn_fwd_fp8_block_sparse.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, F, F, F, I, I,
                                                   ctypes.POINTER(ModParams), ctypes.POINTER(BlockMaskC), P, SZ, P]
    lib.flex_attn_fwd_fp8_block_sparse.restype = I
    lib.flex_attn_bwd_workspace_size.argtypes = [I, I, I]
    lib.flex_attn_bwd_workspace_size.restype = SZ
    lib.flex_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, ctypes.POINTER(ModParams), I,
                                  P, SZ, P]
    lib.flex_attn_bwd.restype = I
    lib.flex_attn_bwd_block_sparse_workspace_size.argtypes = [I, I, I, I, I]
    lib.flex_attn_bwd_block_sparse_workspace_size.restype = SZ
    lib.flex_attn_bwd_block_sparse.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I,
                                               ctypes.POINTER(ModParams), ctypes.POINTER(BlockMaskC), I, P, SZ, P]
    lib.flex_attn_bwd_block_sparse.restype = I
    lib.flex_attn_decode_workspace_size.argtypes = [I, I, I, I, I]
    lib.flex_attn_decode_workspace_size.restype = SZ
    lib.flex_attn_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, I, P, SZ,
                                     ctypes.POINTER(DecodeParamsC), P]
    lib.flex_attn_decode.restype = I
    lib.flex_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, F, I,
                                             ctypes.POINTER(DecodeParamsC), P]
    lib.flex_attn_decode_noalloc.restype = I
    lib.flex_attn_mask_eval.argtypes = [I, ctypes.POINTER(ModParams), I, I, P, P]
    lib.flex_attn_mask_eval.restype = I
    lib.flex_attn_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P]
    lib.flex_attn_selftest_wait_timeout.restype = I
    lib.flex_attn_tile_sizes.argtypes = [I, ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.flex_attn_tile_sizes.restype = None
    lib.flex_attn_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), I]
    lib.flex_attn_device_status.restype = I
    lib.flex_status_string.argtypes = [I]
    lib.flex_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != 0:
        raise FlexAttnError(f"{what}: {STATUS.get(rc, rc)} (status {rc})")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _cuda_tensor(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise FlexAttnError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise FlexAttnError(f"{name} must be contiguous")


def tile_sizes(D: int = 128):
    lib = load_library()
    bm, bn = ctypes.c_int(), ctypes.c_int()
    lib.flex_attn_tile_sizes(D, ctypes.byref(bm), ctypes.byref(bn))
    return bm.value, bn.value


def _expect(t, name, shape, dtype, device):
    """Checks a tensor argument's shape, dtype and device (a wrong size would make the
    kernels read or write past the allocation)."""
    if not isinstance(t, torch.Tensor):
        raise FlexAttnError(f"{name} must be a tensor")
    if tuple(t.shape) != tuple(shape):
        raise FlexAttnError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise FlexAttnError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise FlexAttnError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise FlexAttnError(f"{name} must be contiguous")


def _check_fwd_shapes(q, k, v, out=None, lse_out=None):
    """Shapes and dtypes of a forward's tensors (no device work)."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise FlexAttnError("q, k, v must be 4-D [B, H, S, D]")
    B, H, Sq, D = q.shape
    Bk, Hkv, Skv, Dk = k.shape
    if Bk != B or Dk != D or tuple(v.shape) != tuple(k.shape) or not (q.dtype == k.dtype == v.dtype):
        raise FlexAttnError("shape/dtype mismatch between q, k, v")
    if q.device != k.device or q.device != v.device:
        raise FlexAttnError("q, k, v must be on one device")
    if q.dtype not in DTYPES:
        raise FlexAttnError(f"unsupported dtype {q.dtype}")
    if out is not None:
        _expect(out, "out", q.shape, q.dtype, q.device)
    if lse_out is not None:
        _expect(lse_out, "lse_out", (B, H, Sq), torch.float32, q.device)
    return B, H, Hkv, Sq, Skv, D


def _fwd_args(q, k, v, scale, return_lse, out, lse_out):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda_tensor(t, n)
    B, H, Hkv, Sq, Skv, D = _check_fwd_shapes(q, k, v, out, lse_out if return_lse else None)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = out if out is not None else torch.empty_like(q)
    lse = None
    if return_lse:
        lse = lse_out if lse_out is not None else torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    return B, H, Hkv, Sq, Skv, D, float(scale), o, lse


def _status_word(status, device):
    """Pointer of a caller's per-call status word: an int32 (or uint32) CUDA tensor of one
    element on the call's device, or None for the shared per-device word."""
    if status is None:
        return None
    _cuda_tensor(status, "status")
    if status.numel() != 1 or status.dtype not in (torch.int32, torch.uint32) or status.device != device:
        raise FlexAttnError("status must be a one-element int32 tensor on the call's device")
    return status.data_ptr()


def _mod_params(B, H, score_mod, mask_mod, window, offset, tile_map, alibi_slopes, doc_offsets,
                doc_offsets_kv, status_ptr=None):
    """ModParams and the score_mod id; the captured tensors are checked, not copied."""
    score = SCORE_MODS[score_mod]
    slopes_ptr = None
    if alibi_slopes is not None:
        if score_mod != "alibi":
            raise FlexAttnError("alibi_slopes go with score_mod='alibi'")
        _cuda_tensor(alibi_slopes, "alibi_slopes")
        if alibi_slopes.dtype != torch.float32 or alibi_slopes.numel() != H:
            raise FlexAttnError("alibi_slopes must be float32 with H entries")
        score, slopes_ptr = SCORE_ALIBI_SLOPES, alibi_slopes.data_ptr()
    oq = okv = None
    n_docs = 0
    if mask_mod in ("document", "document_causal"):
        if doc_offsets is None:
            raise FlexAttnError("document masks need doc_offsets [B, n_docs + 1] (int32, CUDA)")
        for t, n in ((doc_offsets, "doc_offsets"), (doc_offsets_kv, "doc_offsets_kv")):
            if t is None:
                continue
            _cuda_tensor(t, n)
            if t.dtype != torch.int32 or t.dim() != 2 or t.shape[0] != B or t.shape[1] < 1:
                raise FlexAttnError(f"{n} must be int32 [B, n_docs + 1]")
        if doc_offsets_kv is not None and tuple(doc_offsets_kv.shape) != tuple(doc_offsets.shape):
            raise FlexAttnError("doc_offsets_kv must have the shape of doc_offsets")
        oq = doc_offsets.data_ptr()
        okv = None if doc_offsets_kv is None else doc_offsets_kv.data_ptr()
        n_docs = doc_offsets.shape[1] - 1
    mp = ModParams(int(window), int(offset), FLAG_TILE_MAP if tile_map is not None else 0,
                   tile_map.data_ptr() if tile_map is not None else None, slopes_ptr, oq, okv, n_docs, status_ptr)
    return mp, score


def fwd(q, k, v, scale=None, score_mod="none", mask_mod="none", window=0, offset=0,
        return_lse=True, out=None, lse_out=None, tile_map=None, alibi_slopes=None, doc_offsets=None,
        doc_offsets_kv=None, status=None):
    """Flex-attention forward.  q [B,H,Sq,D], k/v [B,Hkv,Skv,D] (bf16 or f16, CUDA).

    Returns (O, LSE) (LSE is None when return_lse is False).  ``tile_map``: optional
    uint8 CUDA tensor of ceil(Sq/BM)*ceil(Skv/BN) bytes that receives the tile classes
    of batch 0 / head 0.  Captured tensors: ``alibi_slopes`` (float32 [H], with
    score_mod="alibi"); ``doc_offsets`` / ``doc_offsets_kv`` (int32 [B, n_docs + 1]
    document boundaries, with mask_mod "document" or "document_causal").  ``status``:
    optional one-element int32 CUDA tensor that receives this call's device status bits.
    """
    lib = load_library()
    B, H, Hkv, Sq, Skv, D, scale, o, lse = _fwd_args(q, k, v, scale, return_lse, out, lse_out)
    mp, score = _mod_params(B, H, score_mod, mask_mod, window, offset, tile_map, alibi_slopes, doc_offsets,
                            doc_offsets_kv, _status_word(status, q.device))
    rc = lib.flex_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Sq, Skv, D,
                           scale, score, MASK_MODS[mask_mod], ctypes.byref(mp),
                           DTYPES[q.dtype], _stream(q.device))
    _check(rc, "flex_attn_fwd")
    return o, lse


def fwd_block_sparse(q, k, v, kv_num_blocks, kv_indices, full_kv_num_blocks=None, full_kv_indices=None,
                     scale=None, score_mod="none", mask_mod="none", window=0, offset=0, return_lse=True,
                     out=None, lse_out=None, tile_map=None, block_size=128, alibi_slopes=None, doc_offsets=None,
                     doc_offsets_kv=None, status=None):
    """Forward with a block mask (flex_attn_fwd_block_sparse).  The block lists are int32
    CUDA tensors: counts [Bm, Hm, ceil(Sq/128)], indices [Bm, Hm, ceil(Sq/128), max_blocks],
    Bm in {1, B}, Hm in {1, H}; either (counts, indices) pair may be None, not both.
    Partial blocks apply mask_mod, full blocks only the key-length rule."""
    lib = load_library()
    B, H, Hkv, Sq, Skv, D, scale, o, lse = _fwd_args(q, k, v, scale, return_lse, out, lse_out)
    bm = _block_mask(kv_num_blocks, kv_indices, full_kv_num_blocks, full_kv_indices, Sq, block_size)
    mp, score = _mod_params(B, H, score_mod, mask_mod, window, offset, tile_map, alibi_slopes, doc_offsets,
                            doc_offsets_kv, _status_word(status, q.device))
    rc = lib.flex_attn_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Sq, Skv, D,
                                        scale, score, MASK_MODS[mask_mod], ctypes.byref(mp),
                                        ctypes.byref(bm), DTYPES[q.dtype], _stream(q.device))
    _check(rc, "flex_attn_fwd_block_sparse")
    return o, lse


def _block_mask(kv_num_blocks, kv_indices, full_kv_num_blocks, full_kv_indices, Sq, block_size):
    """BlockMaskC of the lists (int32 CUDA tensors, checked here)."""
    pairs = [(kv_num_blocks, kv_indices, "kv"), (full_kv_num_blocks, full_kv_indices, "full_kv")]
    shape = None
    for num, idx, name in pairs:
        if (num is None) != (idx is None):
            raise FlexAttnError(f"{name}_num_blocks and {name}_indices go together")
        if num is None:
            continue
        _cuda_tensor(num, f"{name}_num_blocks")
        _cuda_tensor(idx, f"{name}_indices")
        if num.dtype != torch.int32 or idx.dtype != torch.int32:
            raise FlexAttnError("block mask tensors must be int32")
        if num.dim() != 3 or idx.dim() != 4 or tuple(idx.shape[:3]) != tuple(num.shape):
            raise FlexAttnError("block mask shapes: counts [Bm, Hm, nq], indices [Bm, Hm, nq, max_blocks]")
        if shape is not None and tuple(idx.shape) != shape:
            raise FlexAttnError("partial and full block lists differ in shape")
        shape = tuple(idx.shape)
    if shape is None:
        raise FlexAttnError("a block mask needs the partial or the full lists")
    bm = BlockMaskC(_ptr(kv_num_blocks), _ptr(kv_indices), _ptr(full_kv_num_blocks), _ptr(full_kv_indices),
                    shape[3], shape[0], shape[1], int(block_size), int(block_size))
    if shape[2] != -(-Sq // 128):
        raise FlexAttnError(f"block mask has {shape[2]} query tiles, Sq={Sq} needs {-(-Sq // 128)}")
    return bm


def fwd_fp8(q8, k8, v8, descale_q=1.0, descale_k=1.0, descale_v=1.0, scale=None, score_mod="none",
            mask_mod="none", window=0, offset=0, alibi_slopes=None, return_lse=True, out=None, lse_out=None,
            workspace=None, status=None, tile_map=None, doc_offsets=None, doc_offsets_kv=None):
    """8-bit forward (flex_attn_fwd_fp8): q8/k8/v8 are torch.float8_e4m3fn CUDA tensors in
    the layouts of fwd(); their values are descale_* times the codes.  Returns (O, LSE)
    with O in bf16.  Head dim 64 or 128.  Mods, captured tensors and tile_map as fwd()."""
    return _fp8(None, q8, k8, v8, descale_q, descale_k, descale_v, scale, score_mod, mask_mod, window, offset,
                alibi_slopes, return_lse, out, lse_out, workspace, status, tile_map, doc_offsets, doc_offsets_kv)


def fwd_fp8_block_sparse(q8, k8, v8, kv_num_blocks, kv_indices, full_kv_num_blocks=None, full_kv_indices=None,
                         descale_q=1.0, descale_k=1.0, descale_v=1.0, scale=None, score_mod="none", mask_mod="none",
                         window=0, offset=0, alibi_slopes=None, return_lse=True, out=None, lse_out=None,
                         workspace=None, status=None, tile_map=None, doc_offsets=None, doc_offsets_kv=None,
                         block_size=128):
    """fwd_fp8 with a block mask (flex_attn_fwd_fp8_block_sparse); the lists as for
    fwd_block_sparse()."""
    bm = _block_mask(kv_num_blocks, kv_indices, full_kv_num_blocks, full_kv_indices, q8.shape[2], block_size)
    return _fp8(bm, q8, k8, v8, descale_q, descale_k, descale_v, scale, score_mod, mask_mod, window, offset,
                alibi_slopes, return_lse, out, lse_out, workspace, status, tile_map, doc_offsets, doc_offsets_kv)


def _fp8(bm, q8, k8, v8, descale_q, descale_k, descale_v, scale, score_mod, mask_mod, window, offset, alibi_slopes,
         return_lse, out, lse_out, workspace, status, tile_map, doc_offsets, doc_offsets_kv):
    lib = load_library()
    for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _cuda_tensor(t, n)
        if t.dtype != torch.float8_e4m3fn:
            raise FlexAttnError(f"{n} must be torch.float8_e4m3fn")
    if q8.dim() != 4 or k8.dim() != 4:
        raise FlexAttnError("q8, k8, v8 must be 4-D [B, H, S, D]")
    B, H, Sq, D = q8.shape
    Bk, Hkv, Skv, Dk = k8.shape
    if Bk != B or Dk != D or tuple(v8.shape) != tuple(k8.shape):
        raise FlexAttnError("shape mismatch between q8, k8, v8")
    if k8.device != q8.device or v8.device != q8.device:
        raise FlexAttnError("q8, k8, v8 must be on one device")
    if out is not None:
        _expect(out, "out", (B, H, Sq, D), torch.bfloat16, q8.device)
    if return_lse and lse_out is not None:
        _expect(lse_out, "lse_out", (B, H, Sq), torch.float32, q8.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = out if out is not None else torch.empty((B, H, Sq, D), dtype=torch.bfloat16, device=q8.device)
    lse = None
    if return_lse:
        lse = lse_out if lse_out is not None else torch.empty((B, H, Sq), dtype=torch.float32, device=q8.device)
    need = int(lib.flex_attn_fwd_fp8_workspace_size(B, Hkv, Skv, D))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q8.device)
    elif workspace.device != q8.device or not workspace.is_contiguous():
        raise FlexAttnError("workspace must be a contiguous tensor on q8's device")
    mp, score = _mod_params(B, H, score_mod, mask_mod, window, offset, tile_map, alibi_slopes, doc_offsets,
                            doc_offsets_kv, _status_word(status, q8.device))
    args = (_ptr(q8), _ptr(k8), _ptr(v8), _ptr(o), _ptr(lse), B, H, Hkv, Sq, Skv, D, float(scale),
            float(descale_q), float(descale_k), float(descale_v), score, MASK_MODS[mask_mod], ctypes.byref(mp))
    tail = (_ptr(workspace), workspace.numel() * workspace.element_size(), _stream(q8.device))
    if bm is None:
        _check(lib.flex_attn_fwd_fp8(*args, *tail), "flex_attn_fwd_fp8")
    else:
        _check(lib.flex_attn_fwd_fp8_block_sparse(*args, ctypes.byref(bm), *tail), "flex_attn_fwd_fp8_block_sparse")
    return o, lse


def fwd_host_workspace_size(B, H, Hkv, Sq, Skv, D) -> int:
    return int(load_library().flex_attn_fwd_host_workspace_size(B, H, Hkv, Sq, Skv, D))


def fwd_host(q, k, v, scale=None, score_mod="none", mask_mod="none", window=0, offset=0, return_lse=True,
             out=None, lse_out=None, alibi_slopes=None, doc_offsets=None, doc_offsets_kv=None, status=None,
             workspace=None, device=None):
    """The forward on HOST tensors (flex_attn_fwd_host): q [B,H,Sq,D], k/v [B,Hkv,Skv,D] CPU
    tensors (pinned memory lets the copies overlap the kernels), results in host tensors
    (``out`` / ``lse_out``, allocated pinned when not given).  The library copies chunks of
    kv heads to ``device`` (default: the current CUDA device) and back while it computes
    the previous ones.  Captured tensors and ``status`` are CUDA tensors as in fwd;
    ``workspace``: optional device buffer of fwd_host_workspace_size bytes.  Returns
    (O, LSE) once the results are in host memory (the call synchronises its stream)."""
    lib = load_library()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or not t.is_contiguous():
            raise FlexAttnError(f"{n} must be a contiguous CPU tensor")
    B, H, Hkv, Sq, Skv, D = _check_fwd_shapes(q, k, v, out, lse_out if return_lse else None)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = out if out is not None else torch.empty(q.shape, dtype=q.dtype).pin_memory()
    lse = None
    if return_lse:
        lse = lse_out if lse_out is not None else torch.empty((B, H, Sq), dtype=torch.float32).pin_memory()
    for t, n in ((o, "out"), (lse, "lse_out")):
        if t is not None and not t.is_contiguous():
            raise FlexAttnError(f"{n} must be contiguous")
    need = fwd_host_workspace_size(B, H, Hkv, Sq, Skv, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    elif (not workspace.is_cuda or workspace.device != dev or not workspace.is_contiguous()
          or workspace.numel() * workspace.element_size() < need):
        raise FlexAttnError(f"workspace must be a contiguous CUDA tensor of at least {need} bytes on {dev}")
    mp, score = _mod_params(B, H, score_mod, mask_mod, window, offset, None, alibi_slopes, doc_offsets,
                            doc_offsets_kv, _status_word(status, dev))
    with torch.cuda.device(dev):
        stream = _stream(dev)
        rc = lib.flex_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Hkv, Sq, Skv, D,
                                    float(scale), score, MASK_MODS[mask_mod], ctypes.byref(mp), DTYPES[q.dtype],
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), stream)
        _check(rc, "flex_attn_fwd_host")
        torch.cuda.current_stream(dev).synchronize()
    return o, lse


def bwd_workspace_size(B, H, Sq) -> int:
    return int(load_library().flex_attn_bwd_workspace_size(B, H, Sq))


def bwd(q, k, v, o, lse, dout, scale=None, score_mod="none", mask_mod="none", window=0, offset=0,
        alibi_slopes=None, doc_offsets=None, doc_offsets_kv=None, dq=None, dk=None, dv=None, workspace=None,
        status=None):
    """Flex-attention backward (flex_attn_bwd): gradients (dq, dk, dv) of sum(dout * o)
    for the forward with the same arguments; o and lse are that forward's outputs.
    dk/dv are [B, Hkv, Skv, D] (summed over the query heads of each group)."""
    return _bwd(None, q, k, v, o, lse, dout, scale, score_mod, mask_mod, window, offset, alibi_slopes, doc_offsets,
                doc_offsets_kv, dq, dk, dv, workspace, status)


def bwd_block_sparse(q, k, v, o, lse, dout, kv_num_blocks, kv_indices, full_kv_num_blocks=None,
                     full_kv_indices=None, scale=None, score_mod="none", mask_mod="none", window=0, offset=0,
                     alibi_slopes=None, doc_offsets=None, doc_offsets_kv=None, dq=None, dk=None, dv=None,
                     workspace=None, status=None, block_size=128):
    """Backward of fwd_block_sparse (flex_attn_bwd_block_sparse): the lists and the other
    arguments as there, o and lse that forward's outputs."""
    bm = _block_mask(kv_num_blocks, kv_indices, full_kv_num_blocks, full_kv_indices, q.shape[2], block_size)
    return _bwd(bm, q, k, v, o, lse, dout, scale, score_mod, mask_mod, window, offset, alibi_slopes, doc_offsets,
                doc_offsets_kv, dq, dk, dv, workspace, status)


def _bwd(bm, q, k, v, o, lse, dout, scale, score_mod, mask_mod, window, offset, alibi_slopes, doc_offsets,
         doc_offsets_kv, dq, dk, dv, workspace, status):
    lib = load_library()
    for t, n in ((o, "o"), (dout, "dout"), (lse, "lse")):
        _cuda_tensor(t, n)
    B, H, Hkv, Sq, Skv, D, scale, _, _ = _fwd_args(q, k, v, scale, False, q, None)
    _expect(o, "o", q.shape, q.dtype, q.device)
    _expect(dout, "dout", q.shape, q.dtype, q.device)
    _expect(lse, "lse", (B, H, Sq), torch.float32, q.device)
    for t, n, like in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        if t is not None:
            _expect(t, n, like.shape, like.dtype, like.device)
    dq = dq if dq is not None else torch.empty_like(q)
    dk = dk if dk is not None else torch.empty_like(k)
    dv = dv if dv is not None else torch.empty_like(v)
    need = bwd_workspace_size(B, H, Sq) if bm is None else int(
        lib.flex_attn_bwd_block_sparse_workspace_size(B, H, Hkv, Sq, Skv))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif workspace.device != q.device or not workspace.is_contiguous():
        raise FlexAttnError("workspace must be a contiguous tensor on q's device")
    mp, score = _mod_params(B, H, score_mod, mask_mod, window, offset, None, alibi_slopes, doc_offsets,
                            doc_offsets_kv, _status_word(status, q.device))
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
            B, H, Hkv, Sq, Skv, D, scale, score, MASK_MODS[mask_mod], ctypes.byref(mp))
    tail = (DTYPES[q.dtype], _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(q.device))
    if bm is None:
        _check(lib.flex_attn_bwd(*args, *tail), "flex_attn_bwd")
    else:
        _check(lib.flex_attn_bwd_block_sparse(*args, ctypes.byref(bm), *tail), "flex_attn_bwd_block_sparse")
    return dq, dk, dv


def decode_workspace_size(B, H, Hkv, cap, D) -> int:
    return int(load_library().flex_attn_decode_workspace_size(B, H, Hkv, cap, D))


def _check_decode_shapes(q, k_cache, v_cache, kv_len, mask=None, out=None, lse_out=None):
    """Shapes, dtypes and devices of a decode's tensors (no device work): a short kv_len
    or mask, a smaller v_cache or a small out would make the kernels read or write past
    the allocation."""
    if q.dim() != 4 or q.shape[2] != 1:
        raise FlexAttnError("decode takes q [B, H, 1, D]")
    B, H, _, D = q.shape
    if q.dtype not in DTYPES:
        raise FlexAttnError(f"unsupported dtype {q.dtype}")
    if k_cache.dim() != 4 or k_cache.shape[0] != B or k_cache.shape[3] != D:
        raise FlexAttnError(f"k_cache must be [B={B}, Hkv, cap, D={D}], got {tuple(k_cache.shape)}")
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    _expect(k_cache, "k_cache", (B, Hkv, cap, D), q.dtype, q.device)
    _expect(v_cache, "v_cache", (B, Hkv, cap, D), q.dtype, q.device)
    _expect(kv_len, "kv_len", (B,), torch.int32, q.device)
    if mask is not None:
        _expect(mask, "mask", (B, H, 1, cap), q.dtype, q.device)
    if out is not None:
        _expect(out, "out", (B, H, 1, D), q.dtype, q.device)
    if lse_out is not None:
        _expect(lse_out, "lse_out", (B, H, 1), torch.float32, q.device)
    return B, H, Hkv, cap, D


def _decode_prep(q, k_cache, v_cache, kv_len, mask, out, lse_out, split_size, status):
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (kv_len, "kv_len")):
        _cuda_tensor(t, n)
    if mask is not None:
        _cuda_tensor(mask, "mask")
    B, H, Hkv, cap, D = _check_decode_shapes(q, k_cache, v_cache, kv_len, mask, out, lse_out)
    o = out if out is not None else torch.empty_like(q)
    lse = lse_out if lse_out is not None else torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    dp = DecodeParamsC(int(split_size), _status_word(status, q.device))
    return B, H, Hkv, cap, D, o, lse, dp


def decode(q, k_cache, v_cache, kv_len, scale, mask=None, out=None, lse_out=None, workspace=None, split_size=0,
           status=None):
    """Decode attention.  q [B,H,1,D]; caches [B,Hkv,cap,D] of q's dtype; kv_len [B] int32
    (CUDA); mask optional [B,H,1,cap] of q's dtype.  ``split_size``: cache positions per
    split (0 = the library's choice, 128 or 256).  ``status``: optional one-element int32
    CUDA tensor that receives this call's device status bits.  Returns (O [B,H,1,D],
    LSE [B,H,1])."""
    lib = load_library()
    B, H, Hkv, cap, D, o, lse, dp = _decode_prep(q, k_cache, v_cache, kv_len, mask, out, lse_out, split_size,
                                                 status)
    need = decode_workspace_size(B, H, Hkv, cap, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif workspace.device != q.device or not workspace.is_contiguous():
        raise FlexAttnError("workspace must be a contiguous tensor on q's device")
    rc = lib.flex_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(kv_len), _ptr(mask), _ptr(o), _ptr(lse),
                              B, H, Hkv, cap, D, float(scale), DTYPES[q.dtype], _ptr(workspace),
                              workspace.numel() * workspace.element_size(), ctypes.byref(dp), _stream(q.device))
    _check(rc, "flex_attn_decode")
    return o, lse


# Bytes of the scratch array compiled into the library for decode_noalloc.
DECODE_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024


def decode_noalloc(q, k_cache, v_cache, kv_len, scale, mask=None, out=None, lse_out=None, split_size=0,
                   status=None):
    """Decode through flex_attn_decode_noalloc: no workspace argument and no device
    allocation inside the library; it uses the scratch array compiled into the library
    (shared by all calls on a device, so calls must not overlap on the GPU).  Outputs
    are allocated here only when ``out`` / ``lse_out`` are not given."""
    lib = load_library()
    B, H, Hkv, cap, D, o, lse, dp = _decode_prep(q, k_cache, v_cache, kv_len, mask, out, lse_out, split_size,
                                                 status)
    rc = lib.flex_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(kv_len), _ptr(mask), _ptr(o),
                                      _ptr(lse), B, H, Hkv, cap, D, float(scale), DTYPES[q.dtype],
                                      ctypes.byref(dp), _stream(q.device))
    _check(rc, "flex_attn_decode_noalloc")
    return o, lse


def mask_eval(mask_mod, Sq, Skv, window=0, offset=0, device="cuda", doc_offsets=None, doc_offsets_kv=None):
    """uint8 [Sq, Skv] CUDA tensor of the forward kernel's keep decisions (document
    masks: the boundaries of batch 0, int32 [1, n_docs + 1] or [B, n_docs + 1])."""
    lib = load_library()
    keep = torch.empty((Sq, Skv), dtype=torch.uint8, device=device)
    B = 1 if doc_offsets is None else doc_offsets.shape[0]
    mp, _ = _mod_params(B, 1, "none", mask_mod, window, offset, None, None, doc_offsets, doc_offsets_kv)
    rc = lib.flex_attn_mask_eval(MASK_MODS[mask_mod], ctypes.byref(mp), Sq, Skv, _ptr(keep), _stream(keep.device))
    _check(rc, "flex_attn_mask_eval")
    return keep


def selftest_wait_timeout(timeout_us: int, device="cuda"):
    """Runs the failure-detection self-test (a bounded wait on a barrier nothing arrives
    on); afterwards device_status() has bit 8 set."""
    lib = load_library()
    dev = torch.device(device)
    _check(lib.flex_attn_selftest_wait_timeout(int(timeout_us), _stream(dev)), "flex_attn_selftest_wait_timeout")


def device_status(reset: bool = True) -> int:
    """Reads (and clears) the device status word; synchronises the device."""
    lib = load_library()
    v = ctypes.c_uint32(0)
    _check(lib.flex_attn_device_status(ctypes.byref(v), 1 if reset else 0), "flex_attn_device_status")
    return int(v.value)
