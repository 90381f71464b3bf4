"""The allocation-free attention entry point (pkv_paged_attention_decode_noalloc).

It serves callers that may not allocate device memory (their memory is already
reserved by a serving engine, or they run in a hook where cudaMalloc/cudaFree
are not allowed because they can synchronise the device). It must give the
same results as the regular entry point, which gets its split-K workspace from
the caller. This file is collected last on purpose and builds its own problem,
so it passes alone in a fresh process as well as after the other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_322_b200 import binding

pytestmark = pytest.mark.gpu

TOL = 2e-3      # the bf16-input attention tolerance used by the parity tests
# Both entry points run the same kernels on the same inputs, so their outputs
# are compared for bit equality (a tolerance would hide a scratch-reuse bug).


def _problem(seed=21, hq=32, hkv=8, d=128, lens=(3000, 4097, 17, 8191, 1, 600)):
    g = torch.Generator(device="cuda").manual_seed(seed)
    bs = 16
    nblk = [-(-n // bs) for n in lens]
    nb = sum(nblk) + 11
    mb = max(nblk)
    perm = torch.randperm(nb, generator=g, device="cuda").int()
    tables = torch.zeros((len(lens), mb), dtype=torch.int32, device="cuda")
    off = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[off:off + n]
        off += n
    kc = torch.randn((nb, bs, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn((nb, bs, hkv, d), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((len(lens), hq, d), generator=g, device="cuda").to(torch.bfloat16)
    ctx = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return q, kc, vc, tables, ctx, 1.0 / math.sqrt(d), max(lens)


@pytest.mark.parametrize("part", [512, 128])
def test_noalloc_matches_regular_entry_point_twice(part):
    q, kc, vc, tables, ctx, scale, maxlen = _problem()
    need = binding.workspace_bytes(q.shape[0], q.shape[1], kc.shape[2], q.shape[2], 16, tables.shape[1], maxlen, part)
    assert 0 < need <= binding.NOALLOC_SCRATCH_BYTES          # the case really uses the scratch
    ref = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    binding.paged_attention_decode(ref, q, kc, vc, tables, ctx, scale, max_context_len=maxlen, partition_tokens=part)
    for _ in range(2):                                           # two calls in a row share the array
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        binding.paged_attention_decode_noalloc(out, q, kc, vc, tables, ctx, scale, max_context_len=maxlen,
                                               partition_tokens=part)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)


def test_noalloc_persistent_schedule_after_split_k_leftovers():
    """The persistent schedule keeps arrival counters in the scratch array. A
    128-token split-K call first fills the array with partial outputs; the
    persistent call that follows must not read them as counters. Two persistent
    calls in a row, each bit-equal to the regular entry point with its own
    workspace, and within the tolerance of the split-K result."""
    q, kc, vc, tables, ctx, scale, maxlen = _problem(seed=22)
    split = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    binding.paged_attention_decode_noalloc(split, q, kc, vc, tables, ctx, scale, max_context_len=maxlen,
                                           partition_tokens=128)
    need = binding.workspace_bytes(q.shape[0], q.shape[1], kc.shape[2], q.shape[2], 16, tables.shape[1], maxlen,
                                   binding.SCHEDULE_PERSISTENT)
    assert 0 < need <= binding.NOALLOC_SCRATCH_BYTES
    ref = torch.empty_like(split)
    binding.paged_attention_decode(ref, q, kc, vc, tables, ctx, scale, max_context_len=maxlen,
                                   partition_tokens=binding.SCHEDULE_PERSISTENT)
    for _ in range(2):
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        binding.paged_attention_decode_noalloc(out, q, kc, vc, tables, ctx, scale, max_context_len=maxlen,
                                               partition_tokens=binding.SCHEDULE_PERSISTENT)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert torch.equal(out, ref)
    assert (ref - split).abs().max().item() <= TOL


def test_noalloc_with_one_partition():
    """Contexts within one partition: no split-K partials, only the schedule's
    unit list in the array."""
    q, kc, vc, tables, ctx, scale, maxlen = _problem(lens=(5, 40, 300))
    ref = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    binding.paged_attention_decode(ref, q, kc, vc, tables, ctx, scale, max_context_len=maxlen, partition_tokens=512)
    out = torch.empty_like(ref)
    binding.paged_attention_decode_noalloc(out, q, kc, vc, tables, ctx, scale, max_context_len=maxlen,
                                           partition_tokens=512)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = binding.library()
    B, hq, hkv, d, mb = 256, 64, 8, 128, 2048
    need = binding.workspace_bytes(B, hq, hkv, d, 16, mb, mb * 16, 16)
    assert need > binding.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.full((B, hq, d), 7.0, dtype=torch.float32, device="cuda")
    kc = torch.zeros((16, 16, hkv, d), dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros((B, mb), dtype=torch.int32, device="cuda")
    ctx = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = lib.pkv_paged_attention_decode_noalloc(
        out.data_ptr(), 0, q.data_ptr(), kc.data_ptr(), kc.data_ptr(), 1, tables.data_ptr(), ctx.data_ptr(),
        ctypes.c_float(1.0), B, hq, hkv, d, 16, mb, 16, mb * 16, 16, torch.cuda.current_stream().cuda_stream)
    assert st == 2                                               # PKV_ERR_UNSUPPORTED, nothing launched
    torch.cuda.synchronize()
    assert out.eq(7.0).all()
