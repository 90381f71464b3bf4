"""Pins of the oracle's swap (GPU pool <-> CPU pool) against what must hold by
construction: a sequence's logical K/V survive swap-out, reuse of the freed GPU
blocks and swap-in; shared blocks move once; counts and free lists balance;
a swap that does not fit changes nothing (CPU only)."""
import copy
import random

import numpy as np
import pytest

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager

BS, HKV, D = 4, 2, 3


def _pools(nb):
    return (np.full((nb, BS, HKV, D), np.nan), np.full((nb, BS, HKV, D), np.nan))


def _write(bm, kc, vc, seq, n, rng):
    """Allocates seq with n tokens and writes random K/V; returns them."""
    slots = bm.allocate(seq, n)
    k = rng.standard_normal((n, HKV, D))
    v = rng.standard_normal((n, HKV, D))
    ocache.reshape_and_cache(k, v, kc, vc, np.asarray(slots))
    return k, v


def _logical(bm, kc, vc, seq):
    t = bm.tables[seq]
    n = bm.lens[seq]
    return oattn.gather_logical(kc, t, n, BS), oattn.gather_logical(vc, t, n, BS)


def _check_balance(bm):
    """Each pool: counts equal the references in the tables of the sequences
    that live there; free list = exactly the unreferenced blocks."""
    gref = [0] * bm.num_blocks
    cref = [0] * bm.num_cpu_blocks
    for s, t in bm.tables.items():
        for b in t:
            if s in bm.swapped:
                cref[b] += 1
            else:
                gref[b] += 1
    assert gref == bm.ref
    assert cref == bm.cpu_ref
    assert sorted(bm.free) == [b for b in range(bm.num_blocks) if gref[b] == 0]
    assert sorted(bm.cpu_free) == [b for b in range(bm.num_cpu_blocks) if cref[b] == 0]


def test_round_trip_through_reused_gpu_blocks():
    rng = np.random.default_rng(7)
    bm = BlockManager(24, BS, free_order=rng.permutation(24), num_cpu_blocks=16,
                      cpu_free_order=rng.permutation(16))
    kc, vc = _pools(24)
    ck, cv = _pools(16)
    data = {s: _write(bm, kc, vc, s, n, rng) for s, n in (("a", 9), ("b", 4), ("c", 13))}
    out = bm.swap_out(["a", "c"])
    assert out is not None and len(out) == 3 + 4
    ocache.swap_blocks(kc, vc, ck, cv, [g for g, _ in out], [c for _, c in out])
    _check_balance(bm)
    # every free GPU block (the freed ones among them) is reused and overwritten
    other = _write(bm, kc, vc, "d", bm.num_free() * BS, rng)
    assert {b for b, _ in out} <= set(bm.tables["d"])
    k, v = _logical(bm, kc, vc, "d")
    np.testing.assert_array_equal(k, other[0])
    assert bm.swap_in(["a"]) is None              # no room while "d" holds the pool
    bm.free_seq("d")
    back = bm.swap_in(["a", "c"])
    assert back is not None and sorted(c for c, _ in back) == sorted(c for _, c in out)
    ocache.swap_blocks(ck, cv, kc, vc, [c for c, _ in back], [g for _, g in back])
    _check_balance(bm)
    for s in ("a", "b", "c"):
        k, v = _logical(bm, kc, vc, s)
        np.testing.assert_array_equal(k, data[s][0])
        np.testing.assert_array_equal(v, data[s][1])
    assert bm.num_free() == 24 - (3 + 1 + 4)
    assert len(bm.cpu_free) == 16


def test_shared_blocks_move_once():
    rng = np.random.default_rng(8)
    bm = BlockManager(16, BS, num_cpu_blocks=8)
    kc, vc = _pools(16)
    ck, cv = _pools(8)
    k, v = _write(bm, kc, vc, "p", 10, rng)       # 3 blocks
    bm.fork("p", "q")
    free_before = bm.num_free()
    pairs = bm.swap_out(["p", "q"])
    assert len(pairs) == 3                         # each shared block copied once
    assert [bm.cpu_ref[c] for _, c in pairs] == [2, 2, 2]
    assert bm.num_free() == free_before + 3
    assert bm.tables["p"] == bm.tables["q"] == [c for _, c in pairs]
    _check_balance(bm)
    ocache.swap_blocks(kc, vc, ck, cv, [g for g, _ in pairs], [c for _, c in pairs])
    pairs_in = bm.swap_in(["q", "p"])
    assert len(pairs_in) == 3
    assert [bm.ref[g] for _, g in pairs_in] == [2, 2, 2]
    ocache.swap_blocks(ck, cv, kc, vc, [c for c, _ in pairs_in], [g for _, g in pairs_in])
    for s in ("p", "q"):
        kk, vv = _logical(bm, kc, vc, s)
        np.testing.assert_array_equal(kk, k)
        np.testing.assert_array_equal(vv, v)


def test_partial_group_keeps_blocks_of_the_sequence_left_behind():
    rng = np.random.default_rng(9)
    bm = BlockManager(16, BS, num_cpu_blocks=8)
    kc, vc = _pools(16)
    ck, cv = _pools(8)
    k, v = _write(bm, kc, vc, "p", 8, rng)        # 2 blocks
    bm.fork("p", "q")
    free_before = bm.num_free()
    pairs = bm.swap_out(["q"])
    assert len(pairs) == 2
    assert bm.num_free() == free_before            # p still holds both blocks
    assert [bm.ref[g] for g, _ in pairs] == [1, 1]
    assert [bm.cpu_ref[c] for _, c in pairs] == [1, 1]
    _check_balance(bm)
    ocache.swap_blocks(kc, vc, ck, cv, [g for g, _ in pairs], [c for _, c in pairs])
    back = bm.swap_in(["q"])
    assert {g for _, g in back}.isdisjoint(bm.tables["p"])   # q comes back into fresh blocks
    ocache.swap_blocks(ck, cv, kc, vc, [c for c, _ in back], [g for _, g in back])
    for s in ("p", "q"):
        kk, vv = _logical(bm, kc, vc, s)
        np.testing.assert_array_equal(kk, k)
        np.testing.assert_array_equal(vv, v)


def test_swap_that_does_not_fit_changes_nothing():
    rng = np.random.default_rng(10)
    bm = BlockManager(16, BS, num_cpu_blocks=2)
    kc, vc = _pools(16)
    _write(bm, kc, vc, "a", 9, rng)                # 3 blocks > 2 CPU blocks
    before = copy.deepcopy(bm.__dict__)
    assert bm.swap_out(["a"]) is None
    assert bm.__dict__ == before
    # swap-in that does not fit: fill the GPU pool while "b" is out
    bm2 = BlockManager(4, BS, num_cpu_blocks=4)
    kc2, vc2 = _pools(4)
    _write(bm2, kc2, vc2, "b", 8, rng)
    assert len(bm2.swap_out(["b"])) == 2
    _write(bm2, kc2, vc2, "c", 3 * BS, rng)
    before = copy.deepcopy(bm2.__dict__)
    assert bm2.swap_in(["b"]) is None
    assert bm2.__dict__ == before


def test_swapped_sequence_rules():
    rng = np.random.default_rng(11)
    bm = BlockManager(8, BS, num_cpu_blocks=8)
    kc, vc = _pools(8)
    _write(bm, kc, vc, "a", 5, rng)
    bm.swap_out(["a"])
    for call in (lambda: bm.append_slot("a"), lambda: bm.make_writable("a", 0), lambda: bm.fork("a", "z"),
                 lambda: bm.block_table("a"), lambda: bm.swap_out(["a"])):
        with pytest.raises(ValueError):
            call()
    with pytest.raises(ValueError):
        bm.swap_in(["nope"])
    bm.free_seq("a")
    assert len(bm.cpu_free) == 8 and bm.num_free() == 8
    _check_balance(bm)


def test_random_operation_mix_keeps_pools_balanced():
    """Brute force on small pools: random allocate / append / fork / free /
    swap sequences; after every step the counts balance and every sequence's
    logical K/V equal what was written into it."""
    rng = np.random.default_rng(12)
    pyr = random.Random(12)
    nb, nc = 32, 24
    bm = BlockManager(nb, BS, free_order=rng.permutation(nb), num_cpu_blocks=nc, cpu_free_order=rng.permutation(nc))
    kc, vc = _pools(nb)
    ck, cv = _pools(nc)
    truth = {}
    next_id = 0
    for _ in range(400):
        op = pyr.choice(["alloc", "append", "fork", "free", "out", "in"])
        live = [s for s in truth if s not in bm.swapped]
        out = [s for s in truth if s in bm.swapped]
        if op == "alloc":
            n = pyr.randint(1, 9)
            if -(-n // BS) <= bm.num_free():
                truth[next_id] = _write(bm, kc, vc, next_id, n, rng)
                next_id += 1
        elif op == "append" and live:
            s = pyr.choice(live)
            r = bm.append_slot(s)
            if r is not None:
                slot, cp = r
                if cp is not None:
                    ocache.copy_blocks(kc, vc, [cp[0]], [cp[1]])
                kn = rng.standard_normal((1, HKV, D))
                vn = rng.standard_normal((1, HKV, D))
                ocache.reshape_and_cache(kn, vn, kc, vc, np.asarray([slot]))
                truth[s] = (np.concatenate([truth[s][0], kn]), np.concatenate([truth[s][1], vn]))
        elif op == "fork" and live:
            s = pyr.choice(live)
            bm.fork(s, next_id)
            truth[next_id] = truth[s]
            next_id += 1
        elif op == "free" and truth:
            s = pyr.choice(list(truth))
            bm.free_seq(s)
            del truth[s]
        elif op == "out" and live:
            group = pyr.sample(live, pyr.randint(1, min(3, len(live))))
            pairs = bm.swap_out(group)
            if pairs:
                ocache.swap_blocks(kc, vc, ck, cv, [g for g, _ in pairs], [c for _, c in pairs])
        elif op == "in" and out:
            group = pyr.sample(out, pyr.randint(1, min(3, len(out))))
            pairs = bm.swap_in(group)
            if pairs:
                ocache.swap_blocks(ck, cv, kc, vc, [c for c, _ in pairs], [g for _, g in pairs])
        _check_balance(bm)
        for s, (k, v) in truth.items():
            pk, pv = (ck, cv) if s in bm.swapped else (kc, vc)
            kk, vv = _logical(bm, pk, pv, s)
            np.testing.assert_array_equal(kk, k)
            np.testing.assert_array_equal(vv, v)
