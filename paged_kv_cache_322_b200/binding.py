"""Thin Python binding of libpkv.so (ctypes).

Argument marshalling only: shapes, dtypes and pointers are read from torch
tensors and passed to the C ABI declared in include/pkv.h; every step of the
path runs in the library's CUDA kernels (or, for the block manager, its C++
host code). There is no fallback: if libpkv.so is missing, every call raises.
Build it with `python -m paged_kv_cache_322_b200.build`.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

PKV_F32, PKV_BF16, PKV_FP8_E4M3 = 0, 1, 2
STATUS = {0: "PKV_OK", 1: "PKV_ERR_INVALID_ARG", 2: "PKV_ERR_UNSUPPORTED", 3: "PKV_ERR_CUDA",
          4: "PKV_ERR_DEVICE_BOUNDS", 5: "PKV_ERR_OUT_OF_BLOCKS", 6: "PKV_ERR_DEVICE_TIMEOUT"}


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = STATUS.get(status, str(status))
        super().__init__(f"{what}: {name} ({_lib().pkv_status_string(status).decode()})")


_L = None
_c = ctypes
_vp, _i32, _i64, _f32, _sz = _c.c_void_p, _c.c_int, _c.c_int64, _c.c_float, _c.c_size_t
_pi32, _pi64 = _c.POINTER(_c.c_int32), _c.POINTER(_c.c_int64)

_SIGS = {
    "pkv_status_string": (_c.c_char_p, [_i32]),
    "pkv_paged_attention_decode": (_i32, [_vp, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _f32, _i32, _i32, _i32, _i32,
                                          _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "pkv_paged_attention_decode_noalloc": (_i32, [_vp, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _f32, _i32, _i32, _i32,
                                                  _i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_paged_attention_decode_fp8": (_i32, [_vp, _i32, _vp, _vp, _vp, _f32, _f32, _vp, _vp, _f32, _i32, _i32, _i32,
                                              _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "pkv_reshape_and_cache_fp8": (_i32, [_vp, _vp, _i32, _vp, _vp, _f32, _f32, _vp, _i32, _i32, _i32, _i32, _i32,
                                         _vp]),
    "pkv_paged_attention_workspace_bytes": (_sz, [_i32] * 8),
    "pkv_paged_attention_multi_query_workspace_bytes": (_sz, [_i32] * 10),
    "pkv_paged_attention_multi_query": (_i32, [_vp, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _f32, _i32, _i32, _i32,
                                               _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "pkv_paged_attention_partition_tokens": (_i32, [_i32] * 8),
    "pkv_paged_attention_shared_prefix_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "pkv_paged_attention_decode_shared_prefix": (_i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _i32, _i32,
                                                        _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "pkv_reshape_and_cache": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_copy_blocks": (_i32, [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pkv_swap_blocks": (_i32, [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp]),
    "pkv_get_device_error": (_i32, [_c.POINTER(_c.c_int), _vp]),
    "pkv_test_withhold_copy": (_i32, [_i32, _i32, _c.c_ulonglong]),
    "pkv_step_ctx_create": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _f32,
                                   _c.POINTER(_vp)]),
    "pkv_step_ctx_destroy": (None, [_vp]),
    "pkv_step_ctx_set_timing": (_i32, [_vp, _i32]),
    "pkv_step_ctx_last_timing": (_i32, [_vp, _c.POINTER(_c.c_float)]),
    "pkv_decode_step": (_i32, [_vp, _vp, _pi64, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _i32, _vp, _vp]),
    "pkv_bm_create": (_i32, [_i32, _i32, _pi32, _c.POINTER(_vp)]),
    "pkv_bm_destroy": (None, [_vp]),
    "pkv_bm_allocate": (_i32, [_vp, _i64, _i32, _pi64]),
    "pkv_bm_append_slots": (_i32, [_vp, _pi64, _i32, _pi64, _pi64, _pi64, _c.POINTER(_c.c_int),
                                   _c.POINTER(_c.c_int)]),
    "pkv_bm_make_writable": (_i32, [_vp, _i64, _i32, _pi64, _pi64]),
    "pkv_bm_fork": (_i32, [_vp, _i64, _i64]),
    "pkv_bm_free": (_i32, [_vp, _i64]),
    "pkv_bm_block_tables": (_i32, [_vp, _pi64, _i32, _i32, _pi32, _pi32]),
    "pkv_bm_num_free": (_i32, [_vp]),
    "pkv_bm_ref_count": (_i32, [_vp, _i32]),
    "pkv_bm_seq_len": (_i32, [_vp, _i64]),
    "pkv_bm_block_size": (_i32, [_vp]),
    "pkv_bm_set_host_pool": (_i32, [_vp, _i32, _pi32]),
    "pkv_bm_swap_out": (_i32, [_vp, _pi64, _i32, _pi64, _pi64, _i32, _c.POINTER(_c.c_int)]),
    "pkv_bm_swap_in": (_i32, [_vp, _pi64, _i32, _pi64, _pi64, _i32, _c.POINTER(_c.c_int)]),
    "pkv_bm_num_free_host": (_i32, [_vp]),
    "pkv_bm_host_ref_count": (_i32, [_vp, _i32]),
    "pkv_bm_is_swapped": (_i32, [_vp, _i64]),
}


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m paged_kv_cache_322_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _L = lib
    return _L


def library():
    """The loaded ctypes library (loads it on first use)."""
    return _lib()


def _check(status: int, what: str):
    if status != 0:
        raise PkvError(status, what)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ---------------------------------------------------------------------------
# torch-facing kernel calls
# ---------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    """float32 / bfloat16 tensors; uint8 tensors hold FP8 (e4m3) cache codes."""
    torch = _torch()
    if t.dtype == torch.float32:
        return PKV_F32
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    if t.dtype == torch.uint8:
        return PKV_FP8_E4M3
    raise TypeError(f"unsupported dtype {t.dtype} (float32, bfloat16, or uint8 for FP8 codes)")


def _stream(t, stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    return s.cuda_stream


def _cuda_contig(*ts):
    """CUDA, contiguous, all on one device and that the current one: the library
    launches on the current device, where another GPU's pointer is not valid."""
    dev = None
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors must be on one device ({dev} and {t.device})")
    if dev is not None:
        cur = _torch().cuda.current_device()
        if dev.index != cur:
            raise ValueError(f"tensors are on {dev} but the current device is cuda:{cur} (torch.cuda.set_device)")


def workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                    max_context_len=0, partition_tokens=0) -> int:
    n = _lib().pkv_paged_attention_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                   max_blocks_per_seq, max_context_len, partition_tokens)
    if n == ctypes.c_size_t(-1).value:
        raise PkvError(1, "pkv_paged_attention_workspace_bytes")
    return n


def partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                     max_context_len=0, partition_tokens=0) -> int:
    return _lib().pkv_paged_attention_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                       max_blocks_per_seq, max_context_len, partition_tokens)


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                           max_context_len: int = 0, partition_tokens: int = 0, workspace=None, stream=None):
    """out[s,h] = softmax(scale q[s,h] K_s^T) V_s over the block-table-addressed cache.

    out, q [B, Hq, D]; caches [NB, bs, Hkv, D]; block_tables int32 [B, MB];
    context_lens int32 [B]. `workspace` (uint8 CUDA tensor) is allocated from
    torch's allocator when not given."""
    torch = _torch()
    _cuda_contig(out, q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (B, hq, d):
        raise ValueError("shape mismatch")
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share a dtype")
    mb = block_tables.shape[1]
    need = workspace_bytes(B, hq, hkv, d, bs, mb, max_context_len, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib().pkv_paged_attention_decode(
        out.data_ptr(), _dtype_code(out), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        _dtype_code(k_cache), block_tables.data_ptr(), context_lens.data_ptr(), float(scale), B, hq, hkv, d, bs,
        mb, nb, int(max_context_len), int(partition_tokens), ws_ptr, ws_n, _stream(q, stream))
    _check(st, "pkv_paged_attention_decode")
    return out


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024
SCHEDULE_PERSISTENT = -1          # partition_tokens value of the persistent schedule


def paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                                   max_context_len: int = 0, partition_tokens: int = 0, stream=None):
    """paged_attention_decode without a workspace: the split-K scratch is a fixed
    array inside the library (NOALLOC_SCRATCH_BYTES per GPU), for callers that
    must not allocate device memory. Raises PkvError(PKV_ERR_UNSUPPORTED) when
    the sizes need more scratch than that. Concurrent calls on different
    streams share the array and must be serialised."""
    torch = _torch()
    _cuda_contig(out, q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (B, hq, d):
        raise ValueError("shape mismatch")
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share a dtype")
    st = _lib().pkv_paged_attention_decode_noalloc(
        out.data_ptr(), _dtype_code(out), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        _dtype_code(k_cache), block_tables.data_ptr(), context_lens.data_ptr(), float(scale), B, hq, hkv, d, bs,
        block_tables.shape[1], nb, int(max_context_len), int(partition_tokens), _stream(q, stream))
    _check(st, "pkv_paged_attention_decode_noalloc")
    return out


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, stream=None):
    """Writes k[t], v[t] ([T, Hkv, D]) into cache slot slot_mapping[t] (int64; < 0 skipped)."""
    torch = _torch()
    _cuda_contig(k, v, k_cache, v_cache, slot_mapping)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    nb, bs, hkv, d = k_cache.shape
    T = k.shape[0]
    if tuple(k.shape) != (T, hkv, d) or tuple(v.shape) != (T, hkv, d) or slot_mapping.numel() != T:
        raise ValueError("shape mismatch")
    if not (k.dtype == v.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("k, v and the caches must share a dtype")
    st = _lib().pkv_reshape_and_cache(k.data_ptr(), v.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                      _dtype_code(k_cache), slot_mapping.data_ptr(), T, hkv, d, bs, nb,
                                      _stream(k_cache, stream))
    _check(st, "pkv_reshape_and_cache")


def reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_scale: float, v_scale: float, stream=None):
    """FP8 (e4m3) append: k, v [T, Hkv, D] bf16 or f32 are quantised into uint8
    caches of codes, code = e4m3(x * (1 / scale)), saturating at +-448."""
    torch = _torch()
    _cuda_contig(k, v, k_cache, v_cache, slot_mapping)
    if slot_mapping.dtype != torch.int64 or k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise TypeError("slot_mapping int64, caches uint8 (FP8 codes)")
    nb, bs, hkv, d = k_cache.shape
    T = k.shape[0]
    if tuple(k.shape) != (T, hkv, d) or tuple(v.shape) != (T, hkv, d) or slot_mapping.numel() != T:
        raise ValueError("shape mismatch")
    if k.dtype != v.dtype:
        raise TypeError("k and v must share a dtype")
    st = _lib().pkv_reshape_and_cache_fp8(k.data_ptr(), v.data_ptr(), _dtype_code(k), k_cache.data_ptr(),
                                          v_cache.data_ptr(), float(k_scale), float(v_scale), slot_mapping.data_ptr(),
                                          T, hkv, d, bs, nb, _stream(k_cache, stream))
    _check(st, "pkv_reshape_and_cache_fp8")


def paged_attention_decode_fp8(out, q, k_cache, v_cache, block_tables, context_lens, scale: float, k_scale: float,
                               v_scale: float, max_context_len: int = 0, partition_tokens: int = 0, workspace=None,
                               stream=None):
    """Decode attention over uint8 FP8 caches (K = code value * k_scale, V likewise); q bf16."""
    torch = _torch()
    _cuda_contig(out, q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if q.dtype != torch.bfloat16 or k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise TypeError("q bfloat16, caches uint8 (FP8 codes)")
    B, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (B, hq, d):
        raise ValueError("shape mismatch")
    mb = block_tables.shape[1]
    need = workspace_bytes(B, hq, hkv, d, bs, mb, max_context_len, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib().pkv_paged_attention_decode_fp8(
        out.data_ptr(), _dtype_code(out), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), float(k_scale),
        float(v_scale), block_tables.data_ptr(), context_lens.data_ptr(), float(scale), B, hq, hkv, d, bs, mb, nb,
        int(max_context_len), int(partition_tokens), ws_ptr, ws_n, _stream(q, stream))
    _check(st, "pkv_paged_attention_decode_fp8")
    return out


def copy_blocks(k_cache, v_cache, src, dst, stream=None):
    """cache[dst[i]] = cache[src[i]] for K and V (src, dst int64 CUDA tensors)."""
    torch = _torch()
    _cuda_contig(k_cache, v_cache, src, dst)
    if src.dtype != torch.int64 or dst.dtype != torch.int64 or src.numel() != dst.numel():
        raise TypeError("src and dst must be int64 tensors of equal length")
    nb, bs, hkv, d = k_cache.shape
    st = _lib().pkv_copy_blocks(k_cache.data_ptr(), v_cache.data_ptr(), _dtype_code(k_cache), src.data_ptr(),
                                dst.data_ptr(), src.numel(), bs, hkv, d, nb, _stream(k_cache, stream))
    _check(st, "pkv_copy_blocks")


def multi_query_workspace_bytes(num_seqs, num_tokens, num_q_heads, num_kv_heads, head_dim, block_size,
                                max_blocks_per_seq, max_query_len, max_context_len=0, partition_tokens=0) -> int:
    n = _lib().pkv_paged_attention_multi_query_workspace_bytes(num_seqs, num_tokens, num_q_heads, num_kv_heads,
                                                               head_dim, block_size, max_blocks_per_seq,
                                                               max_query_len, max_context_len, partition_tokens)
    if n == ctypes.c_size_t(-1).value:
        raise PkvError(1, "pkv_paged_attention_multi_query_workspace_bytes")
    return n


def paged_attention_multi_query(out, q, k_cache, v_cache, block_tables, context_lens, query_start, scale: float,
                                max_query_len: int, max_context_len: int = 0, partition_tokens: int = 0,
                                workspace=None, stream=None):
    """Causal multi-query attention: q / out [T, Hq, D] (rows of all sequences,
    sequence s owning rows query_start[s]..query_start[s+1]-1), bf16 caches
    [NB, bs, Hkv, D] already holding the queries' K/V, context_lens counting
    them; query_start int32 [B + 1]."""
    torch = _torch()
    _cuda_contig(out, q, k_cache, v_cache, block_tables, context_lens, query_start)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32 or query_start.dtype != torch.int32:
        raise TypeError("block_tables, context_lens and query_start must be int32")
    T, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    B = context_lens.shape[0]
    if d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (T, hq, d) or \
            query_start.shape[0] != B + 1:
        raise ValueError("shape mismatch")
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share a dtype")
    mb = block_tables.shape[1]
    need = multi_query_workspace_bytes(B, T, hq, hkv, d, bs, mb, max_query_len, max_context_len, partition_tokens)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib().pkv_paged_attention_multi_query(
        out.data_ptr(), _dtype_code(out), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), _dtype_code(k_cache),
        block_tables.data_ptr(), context_lens.data_ptr(), query_start.data_ptr(), float(scale), B, T, hq, hkv, d, bs,
        mb, nb, int(max_query_len), int(max_context_len), int(partition_tokens), ws_ptr, ws_n, _stream(q, stream))
    _check(st, "pkv_paged_attention_multi_query")
    return out


def shared_prefix_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, prefix_tokens) -> int:
    n = _lib().pkv_paged_attention_shared_prefix_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                                 prefix_tokens)
    if n == ctypes.c_size_t(-1).value:
        raise PkvError(1, "pkv_paged_attention_shared_prefix_workspace_bytes")
    return n


def paged_attention_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens, prefix_tokens: int,
                                         scale: float, max_context_len: int, workspace=None, stream=None):
    """Decode attention (the result of paged_attention_decode) for a batch whose
    block tables share their first prefix_tokens / block_size entries: the shared
    blocks are read once for the whole batch (a cascade: prefix, tails, exact
    merge). out, q [B, Hq, D]; bf16 caches [NB, bs, Hkv, D], head_dim 128."""
    torch = _torch()
    _cuda_contig(out, q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, hq, d = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    if d2 != d or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (B, hq, d):
        raise ValueError("shape mismatch")
    if q.dtype != torch.bfloat16 or k_cache.dtype != torch.bfloat16 or v_cache.dtype != torch.bfloat16:
        raise TypeError("q and the caches must be bfloat16")
    need = shared_prefix_workspace_bytes(B, hq, hkv, d, int(prefix_tokens))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = _lib().pkv_paged_attention_decode_shared_prefix(
        out.data_ptr(), _dtype_code(out), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
        block_tables.data_ptr(), context_lens.data_ptr(), int(prefix_tokens), float(scale), B, hq, hkv, d, bs,
        block_tables.shape[1], nb, int(max_context_len), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream(q, stream))
    _check(st, "pkv_paged_attention_decode_shared_prefix")
    return out


def swap_blocks(src_k, src_v, dst_k, dst_v, src, dst, stream=None):
    """dst_pool[dst[i]] = src_pool[src[i]] for K and V between two pools of the
    same block shape: CUDA tensors or page-locked (pin_memory) CPU tensors, e.g.
    device -> host for a swap-out. src, dst: int64 tensors (CUDA or pinned)."""
    torch = _torch()
    for t in (src_k, src_v, dst_k, dst_v, src, dst):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError("swap_blocks takes CUDA tensors or page-locked CPU tensors")
    if src.dtype != torch.int64 or dst.dtype != torch.int64 or src.numel() != dst.numel():
        raise TypeError("src and dst must be int64 tensors of equal length")
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype:
        raise ValueError("both pools must have the same block shape and dtype")
    dev = next((t.device for t in (src_k, dst_k, src, dst) if t.is_cuda), None)
    if dev is None:
        raise ValueError("one side of the swap must be on the device")
    st = stream.cuda_stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
    _, bs, hkv, d = src_k.shape
    with torch.cuda.device(dev):
        r = _lib().pkv_swap_blocks(src_k.data_ptr(), src_v.data_ptr(), src_k.shape[0], dst_k.data_ptr(),
                                   dst_v.data_ptr(), dst_k.shape[0], _dtype_code(src_k), src.data_ptr(),
                                   dst.data_ptr(), src.numel(), bs, hkv, d, st)
    _check(r, "pkv_swap_blocks")


def get_device_error(stream=None) -> int:
    """Reads and clears the current device's error word (synchronises the stream)."""
    torch = _torch()
    code = ctypes.c_int(0)
    s = stream if stream is not None else torch.cuda.current_stream()
    _check(_lib().pkv_get_device_error(ctypes.byref(code), s.cuda_stream), "pkv_get_device_error")
    return code.value


# ---------------------------------------------------------------------------
# host block manager
# ---------------------------------------------------------------------------
WITHHOLD_DECODE, WITHHOLD_MULTI_QUERY_TC = 0, 1


def test_withhold_copy(kernel: int, index: int, wait_limit_ns: int):
    """Test hook: the next launch of `kernel` withholds one copy in its first CTA
    and gives every bounded wait `wait_limit_ns` (see pkv_test_withhold_copy)."""
    _check(_lib().pkv_test_withhold_copy(kernel, index, wait_limit_ns), "pkv_test_withhold_copy")


class BlockManager:
    """The library's C++ block manager (free list, tables, slots, refcounts, CoW)."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self._h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
            if order.size != num_blocks:
                raise ValueError("free_order must list every block")
        _check(_lib().pkv_bm_create(num_blocks, block_size, _ptr(order, ctypes.c_int32) if order is not None else None,
                                    ctypes.byref(self._h)), "pkv_bm_create")
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _L is not None:
            _L.pkv_bm_destroy(h)
            self._h = None

    def allocate(self, seq_id: int, num_tokens: int) -> np.ndarray:
        slots = np.empty(max(num_tokens, 1), dtype=np.int64)
        _check(_lib().pkv_bm_allocate(self._h, seq_id, num_tokens, _ptr(slots, ctypes.c_int64)), "pkv_bm_allocate")
        return slots[:num_tokens]

    def append_slots(self, seq_ids):
        """One decode step for the listed sequences -> (slot_mapping, copy_src, copy_dst)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.empty(max(n, 1), np.int64)
        src = np.empty(max(n, 1), np.int64)
        dst = np.empty(max(n, 1), np.int64)
        nc, nd = ctypes.c_int(0), ctypes.c_int(0)
        st = _lib().pkv_bm_append_slots(self._h, _ptr(ids, ctypes.c_int64), n, _ptr(slots, ctypes.c_int64),
                                        _ptr(src, ctypes.c_int64), _ptr(dst, ctypes.c_int64), ctypes.byref(nc),
                                        ctypes.byref(nd))
        _check(st, "pkv_bm_append_slots")
        return slots[:n], src[:nc.value], dst[:nc.value]

    def make_writable(self, seq_id: int, logical_block: int):
        s, d = ctypes.c_int64(-1), ctypes.c_int64(-1)
        _check(_lib().pkv_bm_make_writable(self._h, seq_id, logical_block, ctypes.byref(s), ctypes.byref(d)),
               "pkv_bm_make_writable")
        return None if s.value < 0 else (s.value, d.value)

    def fork(self, parent: int, child: int):
        _check(_lib().pkv_bm_fork(self._h, parent, child), "pkv_bm_fork")

    def free(self, seq_id: int):
        _check(_lib().pkv_bm_free(self._h, seq_id), "pkv_bm_free")

    def block_tables(self, seq_ids, max_blocks: int):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.zeros((ids.size, max_blocks), np.int32)
        lens = np.zeros(ids.size, np.int32)
        _check(_lib().pkv_bm_block_tables(self._h, _ptr(ids, ctypes.c_int64), ids.size, max_blocks,
                                          _ptr(tables, ctypes.c_int32), _ptr(lens, ctypes.c_int32)),
               "pkv_bm_block_tables")
        return tables, lens

    def num_free(self) -> int:
        return _lib().pkv_bm_num_free(self._h)

    def ref_count(self, block: int) -> int:
        return _lib().pkv_bm_ref_count(self._h, block)

    def seq_len(self, seq_id: int) -> int:
        return _lib().pkv_bm_seq_len(self._h, seq_id)

    # -- swapping ------------------------------------------------------------
    def set_host_pool(self, num_host_blocks: int, free_order=None):
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32)
            if order.size != num_host_blocks:
                raise ValueError("free_order must list every host block")
        _check(_lib().pkv_bm_set_host_pool(self._h, num_host_blocks,
                                           _ptr(order, ctypes.c_int32) if order is not None else None),
               "pkv_bm_set_host_pool")
        self.num_host_blocks = num_host_blocks

    def _swap(self, fn, seq_ids):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        cap = sum(max(0, -(-max(self.seq_len(int(s)), 0) // self.block_size)) for s in ids.tolist())
        a = np.empty(max(cap, 1), np.int64)
        b = np.empty(max(cap, 1), np.int64)
        n = ctypes.c_int(0)
        _check(getattr(_lib(), fn)(self._h, _ptr(ids, ctypes.c_int64), ids.size, _ptr(a, ctypes.c_int64),
                                   _ptr(b, ctypes.c_int64), cap, ctypes.byref(n)), fn)
        return a[:n.value], b[:n.value]

    def swap_out(self, seq_ids):
        """Moves the group to host blocks -> (device_blocks, host_blocks) to copy."""
        return self._swap("pkv_bm_swap_out", seq_ids)

    def swap_in(self, seq_ids):
        """Brings the group back -> (host_blocks, device_blocks) to copy."""
        return self._swap("pkv_bm_swap_in", seq_ids)

    def num_free_host(self) -> int:
        return _lib().pkv_bm_num_free_host(self._h)

    def host_ref_count(self, block: int) -> int:
        return _lib().pkv_bm_host_ref_count(self._h, block)

    def is_swapped(self, seq_id: int) -> bool:
        r = _lib().pkv_bm_is_swapped(self._h, seq_id)
        if r < 0:
            raise KeyError(seq_id)
        return bool(r)


class DecodeStep:
    """The native decode step (pkv_decode_step): block manager append, H2D of the
    step's q / new K,V / metadata from host buffers, copy-on-write copies, KV
    append, attention, D2H of the output -- one C call per step."""

    def __init__(self, bm: BlockManager, k_cache, v_cache, max_seqs: int, num_q_heads: int,
                 max_blocks_per_seq: int, out_dtype, partition_tokens: int = 0, kv_scales=(1.0, 1.0)):
        torch = _torch()
        self.bm, self.k_cache, self.v_cache = bm, k_cache, v_cache
        nb, bs, hkv, d = k_cache.shape
        if bs != bm.block_size:
            raise ValueError("the caches' block size differs from the block manager's")
        self.num_blocks, self.hq, self.hkv, self.d = nb, num_q_heads, hkv, d
        self.partition_tokens = partition_tokens
        self.out_dtype = out_dtype
        self._h = ctypes.c_void_p()
        _check(_lib().pkv_step_ctx_create(max_seqs, num_q_heads, hkv, d, max_blocks_per_seq, bs, _dtype_code(k_cache),
                                          PKV_F32 if out_dtype == torch.float32 else PKV_BF16,
                                          partition_tokens, float(kv_scales[0]), float(kv_scales[1]),
                                          ctypes.byref(self._h)), "pkv_step_ctx_create")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _L is not None:
            _L.pkv_step_ctx_destroy(h)
            self._h = None

    def __call__(self, seq_ids: np.ndarray, q_host, k_host, v_host, out_host, scale: float, stream=None):
        """q_host/k_host/v_host/out_host: CPU tensors (pinned for asynchronous copies).
        Enqueues the step; synchronise the stream before reading out_host."""
        torch = _torch()
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        s = stream if stream is not None else torch.cuda.current_stream(self.k_cache.device)
        st = _lib().pkv_decode_step(self._h, self.bm._h, _ptr(ids, ctypes.c_int64), ids.size, q_host.data_ptr(),
                                    k_host.data_ptr(), v_host.data_ptr(), self.k_cache.data_ptr(),
                                    self.v_cache.data_ptr(), self.num_blocks, float(scale), self.partition_tokens,
                                    out_host.data_ptr(), s.cuda_stream)
        _check(st, "pkv_decode_step")

    def set_timing(self, enable: bool):
        """Phase timing of the following steps (pkv_step_ctx_set_timing)."""
        _check(_lib().pkv_step_ctx_set_timing(self._h, 1 if enable else 0), "pkv_step_ctx_set_timing")

    def last_timing(self) -> dict:
        """Phases of the last timed step in ms: host block manager, H2D, kernels, D2H
        (waits for that step's D2H)."""
        out = (ctypes.c_float * 4)()
        _check(_lib().pkv_step_ctx_last_timing(self._h, out), "pkv_step_ctx_last_timing")
        return {"host_block_manager": out[0], "h2d": out[1], "kernels": out[2], "d2h": out[3]}
