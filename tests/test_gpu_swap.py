"""GPU parity of block swapping (device pool <-> page-locked host pool):
bit-exact against the oracle's block manager and swap copies, through swap-out,
reuse of the freed device blocks by another sequence, and swap-in; attention
after swap-in against the oracle."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem, step_inputs, tolerance

pytestmark = pytest.mark.gpu


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.uint8:
        return t.numpy().astype(np.int32)
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).numpy().astype(np.int32)


def _np_bits(a, dtype):
    if dtype == torch.uint8:
        return np.asarray(a).astype(np.int32)
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == torch.bfloat16:
        return (a.view(np.uint32) >> 16).astype(np.uint16).view(np.int16).astype(np.int32)
    return a.view(np.int32)


def _canon(bits, dtype):
    b = bits.copy()
    if dtype == torch.uint8:
        b[(b & 0x7F) == 0x7F] = 0x7F
    elif dtype == torch.bfloat16:
        b[((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)] = 0x7FC0
    else:
        b[((b & 0x7F800000) == 0x7F800000) & ((b & 0x7FFFFF) != 0)] = 0x7FC00000
    return b


def _same_blocks(dev_pool, ora_pool, ids):
    ids = list(ids)
    if not ids:
        return
    dt = dev_pool.dtype
    got = _canon(_bits(dev_pool[torch.as_tensor(ids, device=dev_pool.device)]), dt)
    exp = _canon(_np_bits(np.stack([np.asarray(ora_pool[i]) for i in ids]), dt), dt)
    assert np.array_equal(got, exp)


def _filler(w, cache, op, seq, n, seed):
    """A new sequence of n tokens written on both sides (same seeded values)."""
    rng = np.random.default_rng(seed)
    dt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    k = rng.standard_normal((n, w.num_kv_heads, w.head_dim), dtype=np.float32)
    v = rng.standard_normal((n, w.num_kv_heads, w.head_dim), dtype=np.float32)
    if dt == torch.bfloat16:
        k, v = wl.bf16_bits_to_f32(wl.round_to_bf16(k)), wl.bf16_bits_to_f32(wl.round_to_bf16(v))
    cache.add_sequence(seq, torch.from_numpy(k).to("cuda", dt), torch.from_numpy(v).to("cuda", dt))
    op._scatter(k, v, np.asarray(op.bm.allocate(seq, n)))


def _scenario(w, groups, host_blocks, dense=False):
    """Swap each group out, fill the freed device blocks with another sequence,
    free it, swap the groups back in (reverse order); check the moved blocks,
    every sequence's blocks, and attention after one decode step."""
    cache, lens = gpu_problem(w, host_blocks=host_blocks)
    op = OracleProblem(w, dense=dense, cpu_blocks=host_blocks)
    dt = cache.k_cache.dtype
    for g in groups:
        pairs = cache.swap_out(g)
        exp = op.bm.swap_out(g)
        assert pairs == exp
        if exp:
            ocache.swap_blocks(op.kc, op.vc, op.kc_host, op.vc_host, [a for a, _ in exp], [b for _, b in exp])
        torch.cuda.synchronize()
        _same_blocks(cache.k_host, op.kc_host, [b for _, b in exp])
        _same_blocks(cache.v_host, op.vc_host, [b for _, b in exp])
    # the freed device blocks are reused by a filler sequence, then released
    n_fill = cache.bm.num_free() * w.block_size
    if n_fill:
        _filler(w, cache, op, 10_000, n_fill, 77)
        cache.free(10_000)
        op.bm.free_seq(10_000)
    for g in reversed(groups):
        pairs = cache.swap_in(g)
        exp = op.bm.swap_in(g)
        assert pairs == exp
        if exp:
            ocache.swap_blocks(op.kc_host, op.vc_host, op.kc, op.vc, [a for a, _ in exp], [b for _, b in exp])
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    for s in range(w.num_seqs):
        t = op.bm.block_table(s)
        _same_blocks(cache.k_cache, op.kc, t)
        _same_blocks(cache.v_cache, op.vc, t)
    if dense:
        for dev_c, ora_c in ((cache.k_cache, op.kc), (cache.v_cache, op.vc), (cache.k_host, op.kc_host),
                             (cache.v_host, op.vc_host)):
            assert np.array_equal(_canon(_bits(dev_c).reshape(-1), dt),
                                  _canon(_np_bits(ora_c, dt).reshape(-1), dt))
    # attention over the swapped-back sequences
    q, kn, vn = step_inputs(w, 0)
    out = cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale)
    exp = op.decode_step(0)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.max(np.abs(out.float().cpu().numpy() - exp)) <= tolerance(w)


def test_swap_tiny_fp32_whole_pools_bit_exact():
    w = wl.WORKLOADS["tiny_fp32"]
    _scenario(w, [[0, 2], [3]], host_blocks=40, dense=True)


def test_swap_shared_prefix_groups():
    """Forked sequences share their prefix blocks: a group moves each shared
    block once; the sequences left behind keep theirs."""
    w = dataclasses.replace(wl.WORKLOADS["shared_prefix"], num_seqs=8, num_blocks=512, lo=16, hi=80)
    _scenario(w, [[1, 2, 3], [5, 0]], host_blocks=300)


def test_swap_fp8_cache():
    w = dataclasses.replace(wl.WORKLOADS["llama2_7b_fp8"], num_seqs=6, num_blocks=1024, lo=100, hi=700)
    _scenario(w, [[0, 1, 4]], host_blocks=200)


def test_swap_full_size_llama2_7b_round_trip():
    """Half of the 64 sequences of the 7B-shaped workload (16384-block pool) out
    and back: every sequence's blocks equal their content before the swap."""
    w = wl.WORKLOADS["llama2_7b"]
    cache, lens = gpu_problem(w, fill_nan=False, host_blocks=3000)
    ids = np.arange(w.num_seqs)
    before = {}
    for s in ids:
        t = torch.as_tensor(cache.bm.block_tables([s], cache.max_blocks_per_seq)[0][0, :-(-int(lens[s]) // 16)],
                            device="cuda", dtype=torch.int64)
        before[s] = (cache.k_cache[t].clone(), cache.v_cache[t].clone())
    group = ids[::2].tolist()
    pairs = cache.swap_out(group)
    assert len(pairs) == sum(-(-int(lens[s]) // 16) for s in group)
    # overwrite every free device block, then swap back
    n = cache.bm.num_free()
    junk = torch.full((n * 16, w.num_kv_heads, w.head_dim), 3.0, dtype=torch.bfloat16, device="cuda")
    cache.add_sequence(99_999, junk, junk)
    cache.free(99_999)
    cache.swap_in(group)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    for s in ids:
        t = torch.as_tensor(cache.bm.block_tables([s], cache.max_blocks_per_seq)[0][0, :-(-int(lens[s]) // 16)],
                            device="cuda", dtype=torch.int64)
        assert torch.equal(cache.k_cache[t], before[s][0]) and torch.equal(cache.v_cache[t], before[s][1])


def test_swap_bounds_and_memory_kinds():
    nb, bs, hkv, d = 8, 16, 2, 64
    dev_k = torch.zeros((nb, bs, hkv, d), dtype=torch.bfloat16, device="cuda")
    dev_v = torch.zeros_like(dev_k)
    host_k = torch.full((nb, bs, hkv, d), 5.0, dtype=torch.bfloat16).pin_memory()
    host_v = torch.full((nb, bs, hkv, d), 6.0, dtype=torch.bfloat16).pin_memory()
    # an out-of-range pair is skipped and flagged; the valid one is copied
    src = torch.tensor([1, 3], dtype=torch.int64, device="cuda")
    dst = torch.tensor([2, nb], dtype=torch.int64, device="cuda")
    binding.swap_blocks(host_k, host_v, dev_k, dev_v, src, dst)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 4          # PKV_ERR_DEVICE_BOUNDS
    assert torch.all(dev_k[2] == 5.0) and torch.all(dev_v[2] == 6.0)
    assert torch.all(dev_k[torch.arange(nb, device="cuda") != 2] == 0)
    # page-locked block ids are accepted as well (read through the mapped address)
    src_h = torch.tensor([2], dtype=torch.int64).pin_memory()
    dst_h = torch.tensor([7], dtype=torch.int64).pin_memory()
    dev_k[2].fill_(9.0)
    binding.swap_blocks(dev_k, dev_v, host_k, host_v, src_h, dst_h)
    torch.cuda.synchronize()
    assert torch.all(host_k[7] == 9.0) and torch.all(host_k[:7] == 5.0)
    # pageable host memory is refused on the host, before any launch
    pageable = np.zeros(nb * bs * hkv * d, dtype=np.uint16)
    lib = binding.library()
    r = lib.pkv_swap_blocks(dev_k.data_ptr(), dev_v.data_ptr(), nb, pageable.ctypes.data, pageable.ctypes.data, nb,
                            binding.PKV_BF16, src.data_ptr(), dst.data_ptr(), 1, bs, hkv, d, None)
    assert r == 1
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
