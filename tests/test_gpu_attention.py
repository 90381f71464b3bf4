"""GPU parity of paged decode attention against the fp64 oracle.

Tolerances: max |gpu - oracle| <= 1e-5 for fp32 caches and <= 2e-3 for bf16
caches (fp32 output, fp32 accumulation). bf16 outputs are compared with the
oracle rounded to bf16, allowing one bf16 ulp of the oracle value plus 2e-3.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem, step_inputs, tolerance

pytestmark = pytest.mark.gpu


def _bf16_ulp(x):
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_bf16_out(got_bf16: torch.Tensor, ref: np.ndarray):
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    ref_r = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(got - ref_r) <= _bf16_ulp(ref) + 2e-3)


# ---------------------------------------------------------------------------
# seeded workloads, reduced to sizes the oracle finishes in seconds
# ---------------------------------------------------------------------------
SMALL = {
    "tiny_fp32": wl.WORKLOADS["tiny_fp32"],
    "llama2_7b": dataclasses.replace(wl.WORKLOADS["llama2_7b"], num_seqs=6, num_blocks=2048),
    "llama2_13b": dataclasses.replace(wl.WORKLOADS["llama2_13b"], num_seqs=4, num_blocks=1024),
    "gqa_70b": dataclasses.replace(wl.WORKLOADS["gqa_70b"], num_seqs=5, num_blocks=4096),
    "long_splitk": dataclasses.replace(wl.WORKLOADS["long_splitk"], num_seqs=6, num_blocks=12288),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("schedule", ["persistent", "partitioned"])
def test_decode_step_matches_oracle(name, out_dtype, schedule):
    """schedule: persistent = the evenly split schedule (partition_tokens -1);
    partitioned = fixed partitions (the workload's, else the library default)."""
    w = SMALL[name]
    part = -1 if schedule == "persistent" else w.partition_tokens
    cache, lens = gpu_problem(w)
    op = OracleProblem(w)
    for step in range(2):
        q, kn, vn = step_inputs(w, step)
        out = cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale, out_dtype=out_dtype,
                                partition_tokens=part)
        ref = op.decode_step(step)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        if out_dtype == torch.float32:
            err = np.abs(out.cpu().numpy().astype(np.float64) - ref).max()
            assert err <= tolerance(w), err
        else:
            check_bf16_out(out, ref)


def test_tiny_listed_lengths_without_append():
    w = wl.WORKLOADS["tiny_fp32"]
    cache, lens = gpu_problem(w)
    op = OracleProblem(w, dense=True)
    q = torch.from_numpy(wl.decode_q(w, 0)).cuda()
    tables, plens = cache.block_tables(np.arange(w.num_seqs))
    assert plens.tolist() == [7, 33, 100, 250]
    out = torch.empty_like(q)
    binding.paged_attention_decode(out, q, cache.k_cache, cache.v_cache, torch.from_numpy(tables).cuda(),
                                   torch.from_numpy(plens).cuda(), w.scale)
    ref = op.attend(wl.decode_q(w, 0))
    assert np.abs(out.cpu().numpy() - ref).max() <= 1e-5


# ---------------------------------------------------------------------------
# edge cases: ragged contexts, block and partition boundaries, groups, dims
# ---------------------------------------------------------------------------
EDGE_LENS = [0, 1, 2, 15, 16, 17, 31, 33, 255, 256, 257, 511, 512, 513, 1000]


def _edge_problem(seed, hq, hkv, d, dtype, lens, nb=None, bs=16):
    rng = np.random.default_rng(seed)
    need = sum(-(-n // bs) for n in lens)
    nb = nb or need + 37
    order = rng.permutation(nb).astype(np.int32)
    mb = max(1, max(-(-n // bs) for n in lens))
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    kc = torch.full((nb, bs, hkv, d), float("nan"), dtype=tdt, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    ko = np.full((nb, bs, hkv, d), np.nan, np.float32)
    vo = np.full((nb, bs, hkv, d), np.nan, np.float32)
    pbm = binding.BlockManager(nb, bs, order)
    obm = OracleBM(nb, bs, order)
    for s, n in enumerate(lens):
        k = rng.standard_normal((n, hkv, d), dtype=np.float32)
        v = rng.standard_normal((n, hkv, d), dtype=np.float32)
        if dtype == "bf16":
            k, v = wl.bf16_bits_to_f32(wl.round_to_bf16(k)), wl.bf16_bits_to_f32(wl.round_to_bf16(v))
        ps = pbm.allocate(s, n)
        os_ = obm.allocate(s, n)
        assert ps.tolist() == os_
        if n:
            binding.reshape_and_cache(torch.from_numpy(k).cuda().to(tdt), torch.from_numpy(v).cuda().to(tdt), kc, vc,
                                      torch.from_numpy(ps).cuda())
            ocache.reshape_and_cache(k, v, ko, vo, np.asarray(os_))
    tables, plens = pbm.block_tables(np.arange(len(lens)), mb)
    q = rng.standard_normal((len(lens), hq, d), dtype=np.float32)
    if dtype == "bf16":
        q = wl.bf16_bits_to_f32(wl.round_to_bf16(q))
    otables = [obm.block_table(s) for s in range(len(lens))]
    ref = oattn.paged_attention_decode(q, ko, vo, otables, lens, 1.0 / math.sqrt(d), bs)
    dev = dict(q=torch.from_numpy(q).cuda().to(tdt), kc=kc, vc=vc, tables=torch.from_numpy(tables).cuda(),
               lens=torch.from_numpy(plens).cuda(), scale=1.0 / math.sqrt(d), mb=mb, nb=nb)
    return dev, ref


def _run(dev, out_dtype=torch.float32, partition_tokens=0, max_context_len=0):
    out = torch.empty(dev["q"].shape, dtype=out_dtype, device="cuda")
    binding.paged_attention_decode(out, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"], dev["scale"],
                                   max_context_len=max_context_len, partition_tokens=partition_tokens)
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (8, 2), (16, 2)])
@pytest.mark.parametrize("part", [-1, 0, 16, 64, 512])
def test_edge_contexts(dtype, d, hq, hkv, part):
    """part -1 = persistent schedule; 0 = library-chosen partitions; > 0 = fixed."""
    dev, ref = _edge_problem(hq * 1000 + hkv * 100 + d, hq, hkv, d, dtype, EDGE_LENS)
    out = _run(dev, partition_tokens=part)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.array_equal(got[0], np.zeros_like(got[0]))          # context 0 -> zeros
    tol = 1e-5 if dtype == "f32" else 2e-3
    assert np.abs(got - ref).max() <= tol


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 64])
@pytest.mark.parametrize("part", [0, 16, 64, 512])
def test_group_16_edge_contexts(dtype, d, bs, part):
    """Group 16 (32 query heads on 2 KV heads): bf16 runs two 8-wide tensor-core
    head tiles per KV head, f32 four heads per CUDA-core warp."""
    dev, ref = _edge_problem(16000 + d + bs, 32, 2, d, dtype, EDGE_LENS, bs=bs)
    out = _run(dev, partition_tokens=part)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.array_equal(got[0], np.zeros_like(got[0]))
    assert np.abs(got - ref).max() <= (1e-5 if dtype == "f32" else 2e-3)


def test_group_16_persistent_schedule_is_refused():
    dev, _ = _edge_problem(17, 32, 2, 128, "bf16", [40, 50])
    with pytest.raises(binding.PkvError) as e:
        _run(dev, partition_tokens=-1)
    assert e.value.status == 2


@pytest.mark.parametrize("hq,hkv", [(24, 4), (12, 2), (3, 1)])
def test_groups_outside_the_built_set_are_refused(hq, hkv):
    dev, _ = _edge_problem(18, hq, hkv, 128, "bf16", [40, 50])
    with pytest.raises(binding.PkvError) as e:
        _run(dev)
    assert e.value.status == 2


@pytest.mark.parametrize("nseq", [256, 300])
def test_many_short_sequences_partitioned(nseq):
    """Batches at and above the live-first grid order's sequence limit (256):
    both grid orders over short, mixed lengths with small partitions."""
    rng = np.random.default_rng(nseq)
    lens = [int(x) for x in rng.integers(0, 120, size=nseq)]
    lens[5] = 0
    dev, ref = _edge_problem(19 + nseq, 8, 2, 64, "bf16", lens)
    out = _run(dev, partition_tokens=32)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got[5], np.zeros_like(got[5]))
    assert np.abs(got - ref).max() <= 2e-3


def test_partition_counts_agree():
    dev, ref = _edge_problem(5, 32, 8, 128, "bf16", [3000, 4097, 17, 8191])
    outs = [_run(dev, partition_tokens=p).cpu().numpy() for p in (16, 128, 512, 2048, 8192, 0, -1)]
    for o in outs:
        assert np.abs(o - ref).max() <= 2e-3
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 1e-4


def test_bf16_output():
    dev, ref = _edge_problem(6, 64, 8, 128, "bf16", [1, 300, 1500])
    check_bf16_out(_run(dev, out_dtype=torch.bfloat16), ref)


@pytest.mark.parametrize("part", [256, 0, -1])
def test_permutation_of_physical_blocks_is_bitwise_invariant(part):
    """Moving blocks to other physical ids (and the table with them) changes
    nothing: the reduction order depends only on logical positions."""
    dev, _ = _edge_problem(7, 32, 8, 128, "bf16", [700, 33, 1024])
    out1 = _run(dev, partition_tokens=part)
    nb = dev["nb"]
    perm = torch.from_numpy(np.random.default_rng(8).permutation(nb)).cuda()
    kc2, vc2 = torch.empty_like(dev["kc"]), torch.empty_like(dev["vc"])
    kc2[perm], vc2[perm] = dev["kc"], dev["vc"]
    dev2 = dict(dev, kc=kc2, vc=vc2, tables=perm[dev["tables"].long()].int().contiguous())
    out2 = _run(dev2, partition_tokens=part)
    assert torch.equal(out1, out2)


def test_bad_block_id_is_flagged_not_faulted():
    dev, ref = _edge_problem(9, 8, 8, 128, "bf16", [40, 50])
    tables = dev["tables"].clone()
    tables[0, 1] = dev["nb"] + 5                 # outside the pool
    assert binding.get_device_error() == 0
    out = _run(dict(dev, tables=tables))
    assert binding.get_device_error() == 4
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got[1] - ref[1]).max() <= 2e-3   # the other sequence is untouched


def test_context_beyond_table_is_clamped_and_flagged():
    dev, ref = _edge_problem(10, 8, 8, 64, "f32", [20, 32])
    lens = dev["lens"].clone()
    lens[0] = 10 ** 6
    out = _run(dict(dev, lens=lens))
    assert binding.get_device_error() == 4
    # sequence 0 now reads the unwritten (NaN) tail of its last block; the other is untouched
    assert np.abs(out.cpu().numpy()[1] - ref[1]).max() <= 1e-5


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_persistent_schedule_many_small_and_long_items(seed):
    """Mixed batch: many 1-3 block items (whole segments), zero lengths, and a
    few long items that span many CTAs (pieces merged by the last CTA)."""
    rng = np.random.default_rng(100 + seed)
    lens = list(rng.integers(0, 48, size=40)) + [9000, 1, 20000, 0, 4096] + list(rng.integers(1, 700, size=20))
    dev, ref = _edge_problem(200 + seed, 16, 4, 128, "bf16", lens)
    out = _run(dev, partition_tokens=-1, max_context_len=max(lens))
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 2e-3
    # repeated calls reuse the workspace counters (a new epoch each call)
    ws = torch.empty(binding.workspace_bytes(len(lens), 16, 4, 128, 16, dev["mb"], max(lens), -1),
                     dtype=torch.uint8, device="cuda")
    for _ in range(3):
        out2 = torch.empty_like(out)
        binding.paged_attention_decode(out2, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"],
                                       dev["scale"], max_context_len=max(lens), partition_tokens=-1, workspace=ws)
        assert torch.equal(out2, out)
