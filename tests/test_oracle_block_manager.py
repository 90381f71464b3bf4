"""Pins of the oracle block manager against what the pages fix (CPU only)."""
import json
import os
import random

import pytest

from oracle.block_manager import BlockManager, OutOfBlocks


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def test_seven_token_walkthrough(golden_dir):
    g = _load(golden_dir, "block_table_walkthrough.json")
    bm = BlockManager(g["num_blocks"], g["block_size"], g["free_order"])
    slots = bm.allocate("req", g["prompt_tokens"])
    assert bm.block_table("req") == g["after_prefill"]["table"]
    assert slots == g["after_prefill"]["slots"]
    assert bm.num_free() == g["after_prefill"]["num_free"]
    for step in g["decode"]:
        slot, copy = bm.append_slot("req")
        assert copy is None
        assert slot == step["slot"]
        assert bm.block_table("req") == step["table"]
        assert bm.num_free() == step["num_free"]
        assert bm.slot("req", step["position"]) == step["slot"]


def test_cow_fork_example(golden_dir):
    g = _load(golden_dir, "cow_fork.json")
    bm = BlockManager(g["num_blocks"], g["block_size"], g["free_order"])
    bm.allocate("A1", g["prompt_tokens"])
    bm.fork("A1", "A2")
    for name in ("A1", "A2"):
        assert bm.block_table(name) == g["after_fork"][name]
    for b, r in g["after_fork"]["ref"].items():
        assert bm.ref[int(b)] == r
    for name, key in (("A1", "A1_append"), ("A2", "A2_append")):
        slot, copy = bm.append_slot(name)
        exp = g[key]
        assert slot == exp["slot"]
        assert (list(copy) if copy else None) == exp["copy"]
        assert bm.block_table(name) == exp["table"]
    for b, r in g["ref_after"].items():
        assert bm.ref[int(b)] == r


def test_block_counts_are_ceil(golden_dir):
    g = _load(golden_dir, "page_counts.json")
    for n_tok, n_pages in g["cases"]:
        bm = BlockManager(100, g["block_size"])
        bm.allocate("u", n_tok)
        assert len(bm.block_table("u")) == n_pages


def test_out_of_memory_returns_none():
    bm = BlockManager(2, 4)
    assert bm.allocate("a", 8) is not None
    assert bm.num_free() == 0
    assert bm.append_slot("a") is None          # len 8 % 4 == 0 needs a new block
    assert bm.allocate("b", 1) is None
    bm2 = BlockManager(1, 4)
    bm2.allocate("a", 3)
    bm2.fork("a", "b")
    assert bm2.append_slot("a") is None         # copy-on-write needs a free block
    with pytest.raises(OutOfBlocks):
        bm2.make_writable("a", 0)


def test_free_returns_blocks_to_back_in_table_order():
    bm = BlockManager(6, 2, [5, 4, 3, 2, 1, 0])
    bm.allocate("a", 5)                         # blocks 5, 4, 3
    bm.free_seq("a")
    assert list(bm.free) == [2, 1, 0, 5, 4, 3]


def test_beam_pruning_frees_at_zero():
    # "vLLM PagedAttention 解析" §4.2: pruned candidates release blocks they own
    # alone at once; blocks still referenced stay; the shared root goes last.
    bm = BlockManager(16, 4)
    bm.allocate("root", 4)                      # block 0 (full)
    bm.fork("root", "b1")
    bm.fork("root", "b2")
    for seq in ("b1", "b2"):
        for _ in range(5):
            bm.append_slot(seq)
    root_block = bm.block_table("root")[0]
    assert bm.ref[root_block] == 3
    own_b1 = bm.block_table("b1")[1:]
    bm.free_seq("b1")
    assert all(bm.ref[b] == 0 and b in bm.free for b in own_b1)
    assert bm.ref[root_block] == 2
    bm.free_seq("b2")
    bm.free_seq("root")
    assert bm.ref[root_block] == 0 and bm.num_free() == 16


def _check_invariants(bm):
    used = {}
    for seq, t in bm.tables.items():
        assert len(t) == -(-bm.lens[seq] // bm.block_size)
        for b in t:
            used[b] = used.get(b, 0) + 1
    # reference count == number of table entries naming the block
    for b in range(bm.num_blocks):
        assert bm.ref[b] == used.get(b, 0)
    free = list(bm.free)
    assert len(set(free)) == len(free)
    assert not (set(free) & set(used))
    assert len(free) + len(used) == bm.num_blocks
    # a block written by one sequence's append is private to it: every slot a
    # sequence would write next is in a block with ref 1 after append_slot.


@pytest.mark.parametrize("seed", range(20))
def test_random_fork_append_free_invariants(seed):
    rng = random.Random(seed)
    bs = rng.choice([1, 2, 4, 16])
    bm = BlockManager(64, bs, rng.sample(range(64), 64))
    live, nxt = [], 0
    for _ in range(300):
        op = rng.random()
        if op < 0.2 or not live:
            n = rng.randint(0, 3 * bs)
            if bm.allocate(nxt, n) is not None:
                live.append(nxt)
            nxt += 1
        elif op < 0.35:
            p = rng.choice(live)
            bm.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif op < 0.85:
            s = rng.choice(live)
            before = bm.block_table(s)
            r = bm.append_slot(s)
            if r is not None:
                slot, copy = r
                b = slot // bs
                assert bm.ref[b] == 1                 # the written block is private
                assert bm.block_table(s)[-1] == b
                if copy is not None:
                    assert copy[0] == before[-1] and copy[1] == b
        else:
            s = rng.choice(live)
            bm.free_seq(s)
            live.remove(s)
        _check_invariants(bm)


def test_slots_are_distinct_for_private_tokens():
    # brute force on a tiny pool: every token position of every live sequence
    # maps to a slot; positions written after the last fork are in private
    # blocks, so two different sequences never write the same slot.
    bm = BlockManager(12, 2, list(range(11, -1, -1)))
    bm.allocate("a", 3)
    bm.fork("a", "b")
    written = {}
    for seq in ("a", "b", "a", "b", "a"):
        slot, _ = bm.append_slot(seq)
        assert slot not in written
        written[slot] = seq
    for seq in ("a", "b"):
        n = bm.lens[seq]
        for p in range(n):
            s = bm.slot(seq, p)
            assert 0 <= s < 12 * 2
