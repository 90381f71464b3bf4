"""GPU parity of causal multi-query paged attention (chunked prefill and
speculative verification) against the fp64 oracle: max |gpu - oracle| <= 2e-3
(bf16 inputs, fp32 accumulation, fp32 output); bf16 outputs within one bf16 ulp
of the oracle plus 2e-3."""
import dataclasses
import math
import zlib

import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem
from tests.test_gpu_attention import check_bf16_out

pytestmark = pytest.mark.gpu


def _bf16(x):
    return wl.bf16_bits_to_f32(wl.round_to_bf16(np.asarray(x, np.float32)))


def _mq_problem(seed, hq, hkv, d, bs, ctxs, ns):
    """Caches holding ctxs[s] tokens per sequence (the last ns[s] are the
    queries' own), placed by the library's block manager; the oracle's copy."""
    rng = np.random.default_rng(seed)
    nb = sum(-(-c // bs) for c in ctxs) + 11
    order = rng.permutation(nb).astype(np.int32)
    mb = max(1, max(-(-c // bs) for c in ctxs))
    kc = torch.full((nb, bs, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    ko = np.full((nb, bs, hkv, d), np.nan, np.float32)
    vo = ko.copy()
    pbm, obm = binding.BlockManager(nb, bs, order), OracleBM(nb, bs, order)
    for s, c in enumerate(ctxs):
        k = _bf16(rng.standard_normal((c, hkv, d)))
        v = _bf16(rng.standard_normal((c, hkv, d)))
        ps = pbm.allocate(s, c)
        assert ps.tolist() == obm.allocate(s, c)
        if c:
            binding.reshape_and_cache(torch.from_numpy(k).cuda().bfloat16(), torch.from_numpy(v).cuda().bfloat16(),
                                      kc, vc, torch.from_numpy(ps).cuda())
            ocache.reshape_and_cache(k, v, ko, vo, ps)
    qs = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    q = _bf16(rng.standard_normal((int(qs[-1]), hq, d)))
    tables, lens = pbm.block_tables(np.arange(len(ctxs)), mb)
    ref = oattn.paged_attention_multi_query(q, ko, vo, [obm.block_table(s) for s in range(len(ctxs))], ctxs, qs,
                                            1 / math.sqrt(d), bs)
    dev = dict(q=torch.from_numpy(q).cuda().bfloat16(), kc=kc, vc=vc, tables=torch.from_numpy(tables).cuda(),
               lens=torch.from_numpy(lens).cuda(), qs=torch.from_numpy(qs).cuda(), scale=1 / math.sqrt(d),
               max_q=int(max(ns)) if len(ns) else 0)
    return dev, ref


def _run(dev, out_dtype=torch.float32, part=0, out=None):
    if out is None:
        out = torch.empty(dev["q"].shape, dtype=out_dtype, device="cuda")
    binding.paged_attention_multi_query(out, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"], dev["qs"],
                                        dev["scale"], max_query_len=dev["max_q"], partition_tokens=part)
    return out


CASES = {
    # name: (ctxs, ns)  -- ragged mixes around tiles (16 tokens), row tiles (64 rows) and partitions
    "verify": ([1, 5, 17, 64, 300, 1000], [1, 5, 4, 8, 5, 7]),
    "chunks": ([70, 200, 129, 513], [70, 64, 65, 200]),
    "mixed": ([33, 900, 16, 257, 40], [1, 130, 16, 17, 0]),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("hq,hkv,d", [(4, 4, 128), (8, 2, 128), (16, 2, 64), (8, 2, 64), (16, 4, 128), (32, 2, 128),
                                       (32, 2, 64)])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
@pytest.mark.parametrize("part", [0, 64, 256])
def test_multi_query_matches_oracle(case, hq, hkv, d, bs, part):
    ctxs, ns = CASES[case]
    dev, ref = _mq_problem(zlib.crc32(repr((case, hq, hkv, d, bs)).encode()), hq, hkv, d, bs, ctxs, ns)
    out = _run(dev, part=part)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 2e-3


def test_bf16_output_and_untouched_rows():
    """bf16 output; rows of q that belong to no sequence (after the last
    sequence's rows) are not written."""
    ctxs, ns = [300, 50], [20, 9]
    dev, ref = _mq_problem(3, 16, 2, 128, 16, ctxs, ns)
    extra = 5
    q = torch.cat([dev["q"], torch.zeros((extra,) + tuple(dev["q"].shape[1:]), dtype=torch.bfloat16, device="cuda")])
    out = torch.full(q.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    _run(dict(dev, q=q), out=out)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    check_bf16_out(out[:29], ref)
    assert torch.all(out[29:] == 7.0)


def test_one_query_per_sequence_equals_decode_kernel():
    ctxs = [1, 100, 1025, 4000]
    dev, ref = _mq_problem(4, 32, 8, 128, 16, ctxs, [1, 1, 1, 1])
    mq = _run(dev)
    dec = torch.empty_like(mq)
    binding.paged_attention_decode(dec, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"], dev["scale"])
    torch.cuda.synchronize()
    assert np.abs(mq.cpu().numpy() - ref).max() <= 2e-3
    assert np.abs(dec.cpu().numpy() - ref).max() <= 2e-3


def test_bad_query_counts_are_flagged_not_faulted():
    ctxs, ns = [40, 60], [4, 6]
    dev, ref = _mq_problem(5, 8, 8, 64, 16, ctxs, ns)
    lens = dev["lens"].clone()
    lens[0] = 2                                   # 4 queries but 2 cached tokens: n > c
    out = torch.full(dev["q"].shape, 3.0, device="cuda")
    _run(dict(dev, lens=lens), out=out)
    assert binding.get_device_error() == 4
    got = out.cpu().numpy()
    assert np.all(got[:4] == 3.0)                 # the bad sequence is skipped
    assert np.abs(got[4:] - ref[4:]).max() <= 2e-3


def test_chunked_prefill_and_verify_through_the_engine():
    """New sequences prefilled in chunks of 128 (the last chunk ragged) through
    PagedKVCache.extend, then a 4-token speculative step, then decode; every
    output against the oracle over the same appended K/V."""
    from paged_kv_cache_322_b200.engine import PagedKVCache
    rng = np.random.default_rng(6)
    hq, hkv, d, bs = 32, 8, 128, 16
    prompt = [300, 77, 512]
    nb = 256
    order = rng.permutation(nb)                     # both block managers take the same free order
    cache = PagedKVCache(nb, bs, hkv, d, torch.bfloat16, "cuda", free_order=order, max_blocks_per_seq=48,
                         fill_value=float("nan"))
    obm = OracleBM(nb, bs, order)
    ko = np.full((nb, bs, hkv, d), np.nan, np.float32)
    vo = ko.copy()
    seqs = [0, 1, 2]
    for s in seqs:
        cache.bm.allocate(s, 0)
        obm.allocate(s, 0)
    done = [0, 0, 0]

    def step(counts):
        T = sum(counts)
        k = _bf16(rng.standard_normal((T, hkv, d)))
        v = _bf16(rng.standard_normal((T, hkv, d)))
        q = _bf16(rng.standard_normal((T, hq, d)))
        out = cache.extend(seqs, counts, torch.from_numpy(q).cuda().bfloat16(), torch.from_numpy(k).cuda().bfloat16(),
                           torch.from_numpy(v).cuda().bfloat16(), 1 / math.sqrt(d))
        slots = []
        for s, c in zip(seqs, counts):
            for _ in range(c):
                slot, cp = obm.append_slot(s)
                assert cp is None
                slots.append(slot)
        ocache.reshape_and_cache(k, v, ko, vo, np.asarray(slots))
        qs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        ref = oattn.paged_attention_multi_query(q, ko, vo, [obm.block_table(s) for s in seqs],
                                                [obm.lens[s] for s in seqs], qs, 1 / math.sqrt(d), bs)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3

    while any(done[i] < prompt[i] for i in range(3)):
        counts = [min(128, prompt[i] - done[i]) for i in range(3)]
        step(counts)
        done = [done[i] + counts[i] for i in range(3)]
    step([4, 4, 4])                 # speculative verify of 4 draft tokens
    step([1, 1, 1])                 # a plain decode step


def test_full_size_chunk_sampled():
    """A 512-token chunk for each of 16 sequences of the 7B-shaped workload
    (contexts U[512, 2048] before the chunk): sampled rows against the oracle."""
    w = dataclasses.replace(wl.WORKLOADS["llama2_7b"], num_seqs=16, num_blocks=4096)
    cache, lens = gpu_problem(w, max_new_tokens=512)
    op = OracleProblem(w, keep=[2, 9])
    rng = np.random.default_rng(7)
    n = 512
    T = n * w.num_seqs
    k = _bf16(rng.standard_normal((T, w.num_kv_heads, w.head_dim)))
    v = _bf16(rng.standard_normal((T, w.num_kv_heads, w.head_dim)))
    q = _bf16(rng.standard_normal((T, w.num_q_heads, w.head_dim)))
    out = cache.extend(np.arange(w.num_seqs), [n] * w.num_seqs, torch.from_numpy(q).cuda().bfloat16(),
                       torch.from_numpy(k).cuda().bfloat16(), torch.from_numpy(v).cuda().bfloat16(), w.scale)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    for s in (2, 9):
        slots = [op.bm.append_slot(s)[0] for _ in range(n)]
        ocache.reshape_and_cache(k[s * n:(s + 1) * n], v[s * n:(s + 1) * n], op.kc, op.vc, np.asarray(slots))
        ref = oattn.paged_attention_multi_query(q[s * n:(s + 1) * n], op.kc, op.vc, [op.bm.block_table(s)],
                                                [op.bm.lens[s]], np.array([0, n]), w.scale, w.block_size)
        rows = rng.choice(n, 24, replace=False)
        assert np.abs(got[s * n + rows] - ref[rows]).max() <= 2e-3


@pytest.mark.parametrize("part", [0, 512])
@pytest.mark.parametrize("bs", [16, 32, 64])
def test_gqa_verify_rows_padded_into_tensor_memory_tiles(part, bs):
    """Group 8, five draft tokens: 40 query rows per KV head, run on 128-row
    tcgen05 tiles whose other 88 rows are idle."""
    ctxs, ns = [17, 1000, 2049, 4000], [5, 5, 5, 5]
    dev, ref = _mq_problem(8 + bs, 64, 8, 128, bs, ctxs, ns)
    out = _run(dev, part=part)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3


@pytest.mark.parametrize("bs", [8, 16, 32, 64])
def test_both_kernels_at_every_block_size(bs):
    """The same sequences through the mma.sync kernel (4 query tokens x group 4 =
    16 rows per KV head) and the tcgen05 kernel (64 tokens x group 4 = 256 rows),
    at each block size, against the oracle."""
    ctxs = [129, 1000, 33]
    for ns in ([4, 4, 4], [64, 64, 33]):
        dev, ref = _mq_problem(40 + bs + ns[0], 16, 4, 128, bs, ctxs, ns)
        out = _run(dev)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3


@pytest.mark.parametrize("ctx", [40, 64, 65, 128, 129, 192, 256, 257, 1000])
def test_verify_rows_at_kv_tile_boundaries(ctx):
    """Verify-sized rows (group 8, 4 draft tokens = 32 rows per KV head, the
    tcgen05 kernel) at contexts on both sides of its 128-token KV tiles; bf16
    output as well."""
    dev, ref = _mq_problem(50 + ctx, 64, 8, 128, 16, [ctx, ctx + 7], [4, 4])
    out = _run(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3
    check_bf16_out(_run(dev, out_dtype=torch.bfloat16), ref)


@pytest.mark.parametrize("hq,hkv,ns", [
    (64, 8, [5, 3, 5]),        # 40 rows per KV head (5 draft tokens x group 8)
    (64, 8, [8, 1, 6]),        # 64 rows
    (32, 8, [9, 2, 9]),        # 36 rows, group 4
    (8, 8, [33, 1, 20]),       # 33 rows, group 1
    (64, 8, [8, 8, 9]),        # 72 rows
])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
@pytest.mark.parametrize("part", [0, 256])
def test_verify_sized_rows_on_tcgen05(hq, hkv, ns, bs, part):
    """33-72 rows per KV head (verify-sized: draft tokens x group) on the tcgen05
    kernel, its 128-row tile mostly padding; contexts around its 128-token KV tiles
    and block boundaries, with and without partitions; bf16 output as well."""
    ctxs = [n + c for n, c in zip(ns, [300, 127, 1000])]
    dev, ref = _mq_problem(zlib.crc32(repr((hq, hkv, ns, bs)).encode()), hq, hkv, 128, bs, ctxs, ns)
    out = _run(dev, part=part)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 2e-3
    check_bf16_out(_run(dev, out_dtype=torch.bfloat16, part=part), ref)
