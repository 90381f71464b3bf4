"""Pins of the oracle KV append and block copy (CPU only)."""
import json
import os

import numpy as np

from oracle.block_manager import BlockManager
from oracle.cache_ops import copy_blocks, reshape_and_cache


def _flat_offset(pb, t, h, d, bs, nh, hd):
    # address arithmetic of the kernel sketch in "LLM 推理引擎内部原理" §2.4
    return pb * bs * nh * hd + t * nh * hd + h * hd + d


def test_append_writes_walkthrough_slots(golden_dir):
    with open(os.path.join(golden_dir, "block_table_walkthrough.json")) as f:
        g = json.load(f)
    nb, bs, nh, hd = g["num_blocks"], g["block_size"], 3, 5
    bm = BlockManager(nb, bs, g["free_order"])
    prompt_slots = bm.allocate("req", g["prompt_tokens"])
    dec_slots = [bm.append_slot("req")[0] for _ in g["decode"]]
    slots = prompt_slots + dec_slots
    rng = np.random.default_rng(0)
    k = rng.standard_normal((len(slots), nh, hd))
    v = rng.standard_normal((len(slots), nh, hd))
    sentinel = -12345.0
    kc = np.full((nb, bs, nh, hd), sentinel)
    vc = np.full((nb, bs, nh, hd), sentinel)
    reshape_and_cache(k, v, kc, vc, np.array(slots))
    kf, vf = kc.ravel(), vc.ravel()
    touched = np.zeros(kf.size, bool)
    table = bm.block_table("req")
    for pos in range(len(slots)):
        pb, t = table[pos // bs], pos % bs
        for h in range(nh):
            for d in range(hd):
                o = _flat_offset(pb, t, h, d, bs, nh, hd)
                assert kf[o] == k[pos, h, d] and vf[o] == v[pos, h, d]
                touched[o] = True
    assert np.all(kf[~touched] == sentinel) and np.all(vf[~touched] == sentinel)
    # position 7 ('fathers') is block 1 offset 3, position 8 is block 3 offset 0
    assert np.array_equal(kc[1, 3], k[7]) and np.array_equal(kc[3, 0], k[8])


def test_negative_slot_is_skipped():
    kc = np.zeros((2, 4, 1, 2))
    vc = np.zeros((2, 4, 1, 2))
    k = np.ones((3, 1, 2))
    reshape_and_cache(k, 2 * k, kc, vc, np.array([-1, 5, -7]))
    assert kc[1, 1].tolist() == [[1.0, 1.0]] and vc[1, 1].tolist() == [[2.0, 2.0]]
    assert kc.sum() == 2 and vc.sum() == 4


def test_copy_blocks_cow_example():
    # "vLLM PagedAttention 解析" §4.1: physical block 1 is copied to block 3
    rng = np.random.default_rng(1)
    kc = rng.standard_normal((8, 4, 2, 3))
    vc = rng.standard_normal((8, 4, 2, 3))
    k0, v0 = kc.copy(), vc.copy()
    copy_blocks(kc, vc, [1], [3])
    assert np.array_equal(kc[3], k0[1]) and np.array_equal(vc[3], v0[1])
    keep = [b for b in range(8) if b != 3]
    assert np.array_equal(kc[keep], k0[keep]) and np.array_equal(vc[keep], v0[keep])


def test_copy_blocks_many_pairs_read_before_write():
    rng = np.random.default_rng(2)
    kc = rng.standard_normal((10, 2, 1, 4))
    vc = rng.standard_normal((10, 2, 1, 4))
    k0, v0 = kc.copy(), vc.copy()
    src, dst = [0, 1, 2], [7, 8, 9]
    copy_blocks(kc, vc, np.array(src), np.array(dst))
    for s, d in zip(src, dst):
        assert np.array_equal(kc[d], k0[s]) and np.array_equal(vc[d], v0[s])
    assert np.array_equal(kc[:7], k0[:7])
    # a swap is well defined because sources are read before any write
    copy_blocks(kc, vc, [0, 1], [1, 0])
    assert np.array_equal(kc[1], k0[0]) and np.array_equal(kc[0], k0[1])
