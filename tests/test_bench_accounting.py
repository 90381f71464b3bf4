"""The bench's byte and flop accounting against brute-force counts on small
cases (CPU only): the reported GB/s and TFLOP/s rest on these."""
import argparse

import numpy as np
import pytest

import bench
from paged_kv_cache_322_b200 import workloads as wl


@pytest.mark.parametrize("n,lens", [(1, [1, 5, 40]), (5, [5, 9, 100]), (16, [16, 17, 300]), (3, [3])])
def test_mq_flops_counts_every_visible_pair(n, lens):
    hq, d = 3, 4
    pairs = 0
    for c in lens:
        for i in range(n):
            pairs += (c - n + i) + 1                 # tokens 0 .. position c - n + i
    assert bench.mq_flops(np.array(lens), n, hq, d) == 4 * hq * d * pairs


def test_mq_bytes_and_decode_bytes_agree_for_one_query():
    w = wl.WORKLOADS["llama2_7b"]
    lens = np.array([17, 512, 2049])
    w3 = bench.dataclasses.replace(w, num_seqs=3)
    # decode counts a 4-byte length per sequence that the multi-query launch does not
    assert bench.mq_attention_bytes(lens, 1, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size) == \
        bench.attention_bytes(w3, lens, 2) - 4 * 3


def test_attention_bytes_brute_force():
    w = bench.dataclasses.replace(wl.WORKLOADS["gqa_70b_fp8"], num_seqs=2)
    lens = np.array([1, 33])
    kv = sum(lens) * w.num_kv_heads * w.head_dim * 1 * 2                 # e4m3: one byte per element
    q = 2 * w.num_q_heads * w.head_dim * 2                                # bf16 queries
    out = 2 * w.num_q_heads * w.head_dim * 2                              # bf16 output
    tables = (1 + 3) * 4
    assert bench.attention_bytes(w, lens, 2) == kv + q + out + tables + 4 * 2


def test_block_size_override_keeps_pool_tokens():
    w = wl.WORKLOADS["llama2_7b"]
    args = argparse.Namespace(block_size=64, num_seqs=0, num_blocks=0)
    w2 = bench.override_workload(w, args)
    assert w2.block_size == 64 and w2.num_blocks * 64 == w.num_blocks * w.block_size
    args = argparse.Namespace(block_size=0, num_seqs=8, num_blocks=100)
    w3 = bench.override_workload(w, args)
    assert (w3.num_seqs, w3.num_blocks, w3.block_size) == (8, 100, 16)


def test_fork_copy_lists_match_the_oracle_block_manager():
    """The fork bench's copy lists: one copy per child of every parent whose last
    block is partly filled (a full last block takes a fresh block instead), the
    same pairs as the oracle's block manager under the same operations, and the
    pool back to its size after the children are freed."""
    from oracle.block_manager import BlockManager as OracleBM
    from paged_kv_cache_322_b200 import binding
    lens = [16, 17, 31, 32, 1, 100]
    nb, bs, samples = 64, 16, 3
    order = np.random.default_rng(0).permutation(nb).astype(np.int32)
    bm, obm = binding.BlockManager(nb, bs, order), OracleBM(nb, bs, order)
    for s, c in enumerate(lens):
        bm.allocate(s, c)
        obm.allocate(s, c)
    free0 = bm.num_free()
    for _ in range(3):
        src, dst = bench.fork_pairs(bm, len(lens), samples)
        want = []
        kids = list(range(len(lens), len(lens) * samples))
        for c in kids:
            obm.fork((c - len(lens)) // (samples - 1), c)
        for c in kids:
            _, cp = obm.append_slot(c)
            if cp is not None:
                want.append(cp)
        for c in kids:
            obm.free_seq(c)
        assert list(zip(src.tolist(), dst.tolist())) == [tuple(p) for p in want]
        assert len(want) == (samples - 1) * sum(1 for c in lens if c % bs)
        assert bm.num_free() == free0


def test_reference_arm_line(monkeypatch):
    """`bench.py --impl reference` (the CPU oracle) prints the contract's keys,
    with the workload overrides applied and nothing from the other ranks."""
    orig = bench.cpu_baseline
    monkeypatch.setattr(bench, "cpu_baseline", lambda w, target_s: orig(w, 0.2))
    args = argparse.Namespace(workload="tiny_fp32", steps=2, warmup=1, block_size=0, num_seqs=2, num_blocks=0)
    assert bench.run_reference(args, 1, 1) is None
    r = bench.run_reference(args, 1, 0)
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in r, k
    assert r["impl"] == "reference" and r["value"] > 0 and r["ms_per_step"] > 0 and r["config"]["global_batch"] == 2
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0


@pytest.mark.parametrize("B,maxctx,part,bs", [(64, 2060, 0, 16), (1, 4096, 0, 16), (16, 32768, 512, 16),
                                              (32, 1552, 0, 16), (4000, 4096, 256, 16), (2, 70000, 0, 16),
                                              (8, 300, 64, 8)])
def test_decode_launch_count_matches_the_library_schedule(B, maxctx, part, bs):
    """gpu_launches counts the plan kernel exactly when the library lists units
    longest first — which shows in the workspace it asks for: the unit list at
    its front, before any split-K partials."""
    from paged_kv_cache_322_b200 import binding
    hq, hkv, d = 32, 8, 128
    mb = -(-maxctx // bs)
    pt = binding.partition_tokens(B, hq, hkv, d, bs, mb, maxctx, part)
    ws = binding.workspace_bytes(B, hq, hkv, d, bs, mb, maxctx, part)
    parts = -(-maxctx // pt)
    partials = 0
    if parts > 1:
        rows = B * hq * parts
        partials = (rows * d * 4 + 255) // 256 * 256 + rows * 2 * 4
    plan = ws - partials > 0
    assert bench.decode_launches(B, part, pt, maxctx, bs) == int(plan) + 1 + int(parts > 1)
