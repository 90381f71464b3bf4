"""One layer's paged KV cache on the device plus the host block manager, and
the decode step that runs the whole path in order:

    block manager append (slot mapping, copy-on-write pairs)      [host, C++]
    -> copy_blocks for the copy-on-write pairs                      [CUDA]
    -> reshape_and_cache of the new tokens' K/V into their slots    [CUDA]
    -> paged decode attention over the updated cache                [CUDA]

("vLLM PagedAttention 深度解析" §3.3 decode step: write the new token's KV into
its logical block through the block table, allocate a new block when the last
one is full; §4.1: copy a shared block before writing into it.)

Host metadata (slot mapping, copy lists, block tables, lengths) goes to the
device through pinned staging buffers on the caller's stream. This module only
sequences calls of the C ABI; it computes nothing itself.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding


class PagedKVCache:
    """dtype float32 / bfloat16 caches, or torch.uint8 for an FP8 (e4m3) cache
    with per-tensor scales kv_scales = (k_scale, v_scale); FP8 caches take bf16
    K/V on append and bf16 queries."""

    def __init__(self, num_blocks: int, block_size: int, num_kv_heads: int, head_dim: int,
                 dtype: torch.dtype, device, free_order=None, max_blocks_per_seq: int = 0,
                 fill_value: float | None = None, kv_scales=(1.0, 1.0), host_blocks: int = 0,
                 host_free_order=None):
        self.num_blocks, self.block_size = num_blocks, block_size
        self.num_kv_heads, self.head_dim, self.dtype = num_kv_heads, head_dim, dtype
        self.fp8 = dtype == torch.uint8
        self.kv_scales = (float(kv_scales[0]), float(kv_scales[1]))
        self.device = torch.device(device)
        shape = (num_blocks, block_size, num_kv_heads, head_dim)
        if fill_value is None:
            self.k_cache = torch.empty(shape, dtype=dtype, device=self.device)
            self.v_cache = torch.empty(shape, dtype=dtype, device=self.device)
        else:
            fill = 0x7F if (self.fp8 and fill_value != fill_value) else fill_value    # NaN -> the e4m3 NaN code
            self.k_cache = torch.full(shape, fill, dtype=dtype, device=self.device)
            self.v_cache = torch.full(shape, fill, dtype=dtype, device=self.device)
        self.bm = binding.BlockManager(num_blocks, block_size, free_order)
        # page-locked host pool for swapped-out sequences (same block shape)
        self.host_blocks = int(host_blocks)
        self.k_host = self.v_host = None
        if self.host_blocks:
            hshape = (self.host_blocks,) + shape[1:]
            self.k_host = torch.empty(hshape, dtype=dtype, pin_memory=True)
            self.v_host = torch.empty(hshape, dtype=dtype, pin_memory=True)
            if fill_value is not None:
                self.k_host.fill_(fill)
                self.v_host.fill_(fill)
            self.bm.set_host_pool(self.host_blocks, host_free_order)
        self.max_blocks_per_seq = max_blocks_per_seq or num_blocks
        self._pinned = {}

    # -- staging ---------------------------------------------------------
    def _to_device(self, name: str, arr: np.ndarray, stream=None) -> torch.Tensor:
        """Copies a host array to the device through a reusable pinned buffer."""
        t = torch.from_numpy(np.ascontiguousarray(arr))
        buf = self._pinned.get(name)
        if buf is None or buf.numel() < t.numel() or buf.dtype != t.dtype:
            buf = torch.empty(max(t.numel(), 1), dtype=t.dtype, pin_memory=True)
            self._pinned[name] = buf
        # the previous async copy out of this buffer must be done before reuse
        ev = self._pinned.get(name + "/ev")
        if ev is not None:
            ev.synchronize()
        view = buf[:t.numel()].view(t.shape)
        view.copy_(t)
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            dev = view.to(self.device, non_blocking=True)
            e = torch.cuda.Event()
            e.record(s)
        self._pinned[name + "/ev"] = e
        return dev

    # -- sequences ---------------------------------------------------------
    def add_sequence(self, seq_id: int, k: torch.Tensor, v: torch.Tensor, stream=None):
        """New sequence with prompt K/V [n, Hkv, D] (device tensors): allocates
        its blocks and writes the prompt into them."""
        slots = self.bm.allocate(seq_id, k.shape[0])
        if k.shape[0]:
            self.append(k, v, self._to_device("slots", slots, stream), stream=stream)
        return slots

    def append(self, k, v, slot_mapping, stream=None):
        """reshape_and_cache (quantising for an FP8 cache)."""
        if self.fp8:
            binding.reshape_and_cache_fp8(k, v, self.k_cache, self.v_cache, slot_mapping, *self.kv_scales,
                                          stream=stream)
        else:
            binding.reshape_and_cache(k, v, self.k_cache, self.v_cache, slot_mapping, stream=stream)

    def attention(self, out, q, tables, lens, scale, max_context_len=0, partition_tokens=0, workspace=None,
                  stream=None):
        if self.fp8:
            return binding.paged_attention_decode_fp8(out, q, self.k_cache, self.v_cache, tables, lens, scale,
                                                      *self.kv_scales, max_context_len=max_context_len,
                                                      partition_tokens=partition_tokens, workspace=workspace,
                                                      stream=stream)
        return binding.paged_attention_decode(out, q, self.k_cache, self.v_cache, tables, lens, scale,
                                              max_context_len=max_context_len, partition_tokens=partition_tokens,
                                              workspace=workspace, stream=stream)

    def fork(self, parent: int, child: int):
        self.bm.fork(parent, child)

    def make_writable(self, seq_ids, logical_block: int, stream=None):
        """Copy-on-write of one logical block for each listed sequence; runs the
        copies. Returns the (src, dst) pairs."""
        pairs = [p for p in (self.bm.make_writable(s, logical_block) for s in seq_ids) if p is not None]
        if pairs:
            arr = np.asarray(pairs, dtype=np.int64)
            binding.copy_blocks(self.k_cache, self.v_cache, self._to_device("cow_src", arr[:, 0], stream),
                                self._to_device("cow_dst", arr[:, 1], stream), stream=stream)
        return pairs

    def free(self, seq_id: int):
        self.bm.free(seq_id)

    # -- preemption by swapping ---------------------------------------------
    def swap_out(self, seq_ids, stream=None):
        """Moves a group of sequences' blocks to the host pool and frees their
        device blocks; the copies run on `stream` before anything queued after
        them reuses the blocks. Returns the (device, host) block pairs."""
        if not self.host_blocks:
            raise RuntimeError("no host pool (host_blocks=0)")
        dev_b, host_b = self.bm.swap_out(seq_ids)
        if dev_b.size:
            binding.swap_blocks(self.k_cache, self.v_cache, self.k_host, self.v_host,
                                self._to_device("swap_src", dev_b, stream), self._to_device("swap_dst", host_b, stream),
                                stream=stream)
        return list(zip(dev_b.tolist(), host_b.tolist()))

    def swap_in(self, seq_ids, stream=None):
        """Brings a swapped-out group back into fresh device blocks. Returns the
        (host, device) block pairs."""
        if not self.host_blocks:
            raise RuntimeError("no host pool (host_blocks=0)")
        host_b, dev_b = self.bm.swap_in(seq_ids)
        if dev_b.size:
            binding.swap_blocks(self.k_host, self.v_host, self.k_cache, self.v_cache,
                                self._to_device("swap_src", host_b, stream), self._to_device("swap_dst", dev_b, stream),
                                stream=stream)
        return list(zip(host_b.tolist(), dev_b.tolist()))

    def block_tables(self, seq_ids):
        return self.bm.block_tables(seq_ids, self.max_blocks_per_seq)

    # -- several tokens per sequence: chunked prefill, speculative verify -----
    def extend(self, seq_ids, counts, q, k_new, v_new, scale: float, out=None, out_dtype=torch.float32,
               partition_tokens: int = 0, stream=None):
        """Appends counts[i] tokens to sequence seq_ids[i] (k_new, v_new [T, Hkv, D],
        rows grouped by sequence in the listed order) and returns causal
        attention of their queries q [T, Hq, D] over each sequence's cache."""
        seq_ids = np.asarray(seq_ids, dtype=np.int64)
        counts = np.asarray(counts, dtype=np.int64)
        if seq_ids.shape != counts.shape or (counts < 0).any() or int(counts.sum()) != q.shape[0]:
            raise ValueError("counts must match the rows of q, one count per sequence")
        order = np.repeat(seq_ids, counts)
        slots, src, dst = self.bm.append_slots(order)
        if src.size:
            binding.copy_blocks(self.k_cache, self.v_cache, self._to_device("src", src, stream),
                                self._to_device("dst", dst, stream), stream=stream)
        if order.size:
            self.append(k_new, v_new, self._to_device("slots", slots, stream), stream=stream)
        tables, lens = self.block_tables(seq_ids)
        qs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=self.device)
        if q.shape[0]:
            binding.paged_attention_multi_query(
                out, q, self.k_cache, self.v_cache, self._to_device("tables", tables, stream),
                self._to_device("lens", lens, stream), self._to_device("qstart", qs, stream), scale,
                max_query_len=int(counts.max()), max_context_len=int(lens.max()), partition_tokens=partition_tokens,
                stream=stream)
        return out

    # -- the decode step -----------------------------------------------------
    def decode_step(self, seq_ids, q, k_new, v_new, scale: float, out=None, out_dtype=torch.float32,
                    partition_tokens: int = 0, stream=None):
        """Appends one token per sequence (k_new, v_new [B, Hkv, D]) and returns
        attention of q [B, Hq, D] over each sequence's updated context."""
        seq_ids = np.asarray(seq_ids, dtype=np.int64)
        slots, src, dst = self.bm.append_slots(seq_ids)
        if src.size:
            binding.copy_blocks(self.k_cache, self.v_cache, self._to_device("src", src, stream),
                                self._to_device("dst", dst, stream), stream=stream)
        self.append(k_new, v_new, self._to_device("slots", slots, stream), stream=stream)
        tables, lens = self.block_tables(seq_ids)
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=self.device)
        self.attention(out, q, self._to_device("tables", tables, stream), self._to_device("lens", lens, stream),
                       scale, max_context_len=int(lens.max()) if lens.size else 0, partition_tokens=partition_tokens,
                       stream=stream)
        return out
