"""Oracle cache-side operations: KV append and block copy.

TEST INFRASTRUCTURE (see oracle/__init__.py).

Cache layout, from the kernel sketch in "LLM 推理引擎内部原理" §2.4: each cache
is [num_blocks, block_size, num_kv_heads, head_dim]; token offset t of physical
block pb holds head h's vector at (pb, t, h, :).

- reshape_and_cache: "vLLM PagedAttention 解析" §3.3 (Prefill step ③ and Decode
  step ②): each new token's K and V are written into the physical slot that the
  block table maps its position to. A slot is physical_block * block_size +
  offset ("LLM 推理引擎内部原理" §2.3 append_slot). Negative slots mean "skip"
  (a padding convention of this library; the pages are silent).
- copy_blocks: "vLLM PagedAttention 解析" §4.1: the shared physical block is
  copied to the fresh block, K and V, all block_size slots.

Both work on any array-like cache supporting numpy-style [block] and
[block, offset] indexing and assignment.
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping):
    """Sequential scatter: token t goes to (slot // bs, slot % bs). In place."""
    bs = int(k_cache.shape[1])
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        b, o = divmod(int(slot), bs)
        k_cache[b, o] = k[t]
        v_cache[b, o] = v[t]


def copy_blocks(k_cache, v_cache, src, dst):
    """cache[dst[i]] = cache[src[i]] for every pair, K and V, reading every
    source before writing any destination. In place."""
    src = [int(s) for s in np.asarray(src).tolist()]
    dst = [int(d) for d in np.asarray(dst).tolist()]
    snap_k = [np.array(k_cache[s], copy=True) for s in src]
    snap_v = [np.array(v_cache[s], copy=True) for s in src]
    for i, d in enumerate(dst):
        k_cache[d] = snap_k[i]
        v_cache[d] = snap_v[i]


def swap_blocks(src_k, src_v, dst_k, dst_v, src, dst):
    """dst_pool[dst[i]] = src_pool[src[i]] for every pair, K and V: the block
    moves of a swap between the GPU pool and the CPU pool ("vLLM PagedAttention
    深度解析" §5.2 Swapping; "LLM 推理引擎内部原理" §3.1 blocks_to_swap_in/out).
    The two pools are different arrays, so pairs cannot alias. In place on dst."""
    for s, d in zip(np.asarray(src).tolist(), np.asarray(dst).tolist()):
        dst_k[int(d)] = np.array(src_k[int(s)], copy=True)
        dst_v[int(d)] = np.array(src_v[int(s)], copy=True)


def reshape_and_cache_fp8(k, v, k_codes, v_codes, slot_mapping, k_scale: float, v_scale: float):
    """KV append into an FP8 (e4m3) cache: token t's K (V) is stored as the
    codes of float32(k[t] * inv_scale) (see oracle.fp8). Caches hold uint8 codes."""
    from oracle import fp8
    bs = int(k_codes.shape[1])
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        b, o = divmod(int(slot), bs)
        k_codes[b, o] = fp8.quantize(k[t], k_scale)
        v_codes[b, o] = fp8.quantize(v[t], v_scale)
