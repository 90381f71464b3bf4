"""Test harness: builds the same decode problem twice from the seeded inputs,
once with the oracle (CPU, fp64) and once through the library (GPU), each side
with its own block manager. Nothing here computes attention or addresses."""
from __future__ import annotations

import numpy as np

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_322_b200 import workloads as wl


class SparsePool:
    """A cache [num_blocks, bs, Hkv, D] that stores only written blocks; unwritten
    blocks read as NaN (like the sentinel-filled device pool; the NaN code 0x7F
    for an FP8 pool of uint8 codes)."""

    def __init__(self, num_blocks, bs, hkv, d, dtype=np.float32):
        self.shape = (num_blocks, bs, hkv, d)
        self.dtype = dtype
        self.blocks = {}

    def _blk(self, b):
        b = int(b)
        if b not in self.blocks:
            fill = 0x7F if self.dtype == np.uint8 else np.nan
            self.blocks[b] = np.full(self.shape[1:], fill, dtype=self.dtype)
        return self.blocks[b]

    def __getitem__(self, key):
        if isinstance(key, tuple):
            return self._blk(key[0])[key[1]]
        if isinstance(key, (int, np.integer)):
            return self._blk(key)
        return np.stack([self._blk(b) for b in np.asarray(key).tolist()]) if len(key) else \
            np.zeros((0,) + self.shape[1:], self.dtype)

    def __setitem__(self, key, val):
        if isinstance(key, tuple):
            self._blk(key[0])[key[1]] = val
        else:
            self._blk(key)[...] = val


class OracleProblem:
    """Oracle side of a workload: block tables from the oracle block manager,
    cache contents for the listed sequences only (`keep`, default all)."""

    def __init__(self, w: wl.Workload, keep=None, dense=False, cpu_blocks=0):
        self.w = w
        self.lens = wl.context_lens(w)
        self.bm = OracleBM(w.num_blocks, w.block_size, wl.free_order(w), num_cpu_blocks=cpu_blocks)
        shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
        self.fp8 = w.kv_dtype == "fp8"
        dt, fill = (np.uint8, 0x7F) if self.fp8 else (np.float32, np.nan)
        if dense:
            self.kc = np.full(shape, fill, dt)
            self.vc = np.full(shape, fill, dt)
        else:
            self.kc = SparsePool(*shape, dtype=dt)
            self.vc = SparsePool(*shape, dtype=dt)
        hshape = (cpu_blocks,) + shape[1:]
        self.kc_host = np.full(hshape, fill, dt)       # CPU pool of swapped-out blocks
        self.vc_host = np.full(hshape, fill, dt)
        self.keep = set(range(w.num_seqs)) if keep is None else set(int(s) for s in keep)
        if w.ctx == "shared_prefix":
            self._build_shared()
        else:
            for s in range(w.num_seqs):
                slots = self.bm.allocate(s, int(self.lens[s]))
                if s in self.keep:
                    k, v = wl.prompt_kv(w, s, int(self.lens[s]))
                    self._scatter(k, v, np.asarray(slots))
        self.cow_pairs = []

    def _scatter(self, k, v, slots):
        if self.fp8:
            ocache.reshape_and_cache_fp8(k, v, self.kc, self.vc, slots, self.w.kv_scale, self.w.kv_scale)
        else:
            ocache.reshape_and_cache(k, v, self.kc, self.vc, slots)

    def _build_shared(self):
        w = self.w
        p = w.shared_prefix
        slots = self.bm.allocate(-1, p)
        k0, v0 = wl.prompt_kv(w, 0, int(self.lens[0]))
        self._scatter(k0[:p], v0[:p], np.asarray(slots))
        for s in range(w.num_seqs):
            self.bm.fork(-1, s)
        self.bm.free_seq(-1)
        for s in range(w.num_seqs):
            n = int(self.lens[s])
            tail = [self.bm.append_slot(s)[0] for _ in range(n - p)]
            if s in self.keep:
                k, v = wl.prompt_kv(w, s, n)
                self._scatter(k[p:], v[p:], np.asarray(tail))

    def fork_last_shared_block(self):
        """Copy-on-write of the last shared prefix block for every sequence
        (all but the last one copy; the last keeps the original)."""
        last = self.w.shared_prefix // self.w.block_size - 1
        pairs = [self.bm.make_writable(s, last) for s in range(self.w.num_seqs)]
        pairs = [x for x in pairs if x is not None]
        if pairs:
            ocache.copy_blocks(self.kc, self.vc, [a for a, _ in pairs], [b for _, b in pairs])
        self.cow_pairs = pairs
        return pairs

    def decode_step(self, step: int, seqs=None):
        """Appends step `step`'s token to every sequence; returns the fp64
        attention output of the listed sequences (default: kept ones)."""
        w = self.w
        q = wl.decode_q(w, step)
        kn, vn = wl.decode_kv(w, step)
        slots = []
        for s in range(w.num_seqs):
            slot, copy = self.bm.append_slot(s)
            assert copy is None
            slots.append(slot if s in self.keep else -1)
        self._scatter(kn, vn, np.asarray(slots))
        return self.attend(q, seqs)

    def attend(self, q, seqs=None):
        seqs = sorted(self.keep) if seqs is None else list(seqs)
        tables = {s: self.bm.block_table(s) for s in seqs}
        lens = {s: self.bm.lens[s] for s in seqs}
        if self.fp8:
            return oattn.paged_attention_decode_fp8(q, self.kc, self.vc, _TableView(tables), _TableView(lens),
                                                    self.w.scale, self.w.block_size, self.w.kv_scale,
                                                    self.w.kv_scale, seqs=seqs)
        return oattn.paged_attention_decode(q, self.kc, self.vc, _TableView(tables), _TableView(lens),
                                            self.w.scale, self.w.block_size, seqs=seqs)


class _TableView:
    def __init__(self, d):
        self.d = d

    def __getitem__(self, s):
        return self.d[int(s)]


def gpu_problem(w: wl.Workload, device="cuda", fill_nan=True, max_new_tokens=4, host_blocks=0):
    """Library side: a PagedKVCache with the workload's prompts written by
    reshape_and_cache through the library's block manager."""
    import torch
    from paged_kv_cache_322_b200.engine import PagedKVCache
    lens = wl.context_lens(w)
    dt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16          # q / k / v
    cdt = torch.uint8 if w.kv_dtype == "fp8" else dt                        # caches
    mb = -(-int(lens.max() + max_new_tokens) // w.block_size)
    cache = PagedKVCache(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, cdt, device,
                         free_order=wl.free_order(w), max_blocks_per_seq=mb,
                         fill_value=float("nan") if fill_nan else None, kv_scales=(w.kv_scale, w.kv_scale),
                         host_blocks=host_blocks)
    def dev(x):
        return torch.from_numpy(x).to(device=device, dtype=dt)
    if w.ctx == "shared_prefix":
        p = w.shared_prefix
        k0, v0 = wl.prompt_kv(w, 0, int(lens[0]))
        cache.add_sequence(-1, dev(k0[:p]), dev(v0[:p]))
        for s in range(w.num_seqs):
            cache.fork(-1, s)
        cache.free(-1)
        for s in range(w.num_seqs):
            n = int(lens[s])
            k, v = wl.prompt_kv(w, s, n)
            kt, vt = dev(k[p:]), dev(v[p:])
            slots = np.concatenate([cache.bm.append_slots([s])[0] for _ in range(n - p)])
            cache.append(kt, vt, torch.from_numpy(slots).to(device))
    else:
        kvs = wl.prompt_kv_all(w, lens)
        for s in range(w.num_seqs):
            k, v = kvs[s]
            cache.add_sequence(s, dev(k), dev(v))
    return cache, lens


def step_inputs(w: wl.Workload, step: int, device="cuda"):
    import torch
    dt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    q = torch.from_numpy(wl.decode_q(w, step)).to(device=device, dtype=dt)
    kn, vn = wl.decode_kv(w, step)
    return q, torch.from_numpy(kn).to(device=device, dtype=dt), torch.from_numpy(vn).to(device=device, dtype=dt)


def tolerance(w: wl.Workload) -> float:
    """Max abs error allowed against the fp64 oracle: 1e-5 for fp32 inputs,
    2e-3 for bf16-rounded inputs and for FP8 caches (the oracle attends over the
    same dequantised values; fp32 accumulation, fp32 output)."""
    return 1e-5 if w.kv_dtype == "f32" else 2e-3
