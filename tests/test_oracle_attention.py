"""Pins of the oracle paged decode attention (CPU only).

Each pin comes from outside the oracle: a hand-derived worked example, torch's
own fp64 scaled_dot_product_attention over contiguous K/V, closed forms, and
invariance under relabelling of physical blocks.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.block_manager import BlockManager
from oracle.cache_ops import reshape_and_cache
from oracle.paged_attention import paged_attention_decode


def _hand(golden_dir):
    with open(os.path.join(golden_dir, "attention_hand_example.json")) as f:
        return json.load(f)


def test_hand_worked_example(golden_dir):
    g = _hand(golden_dir)
    kc, vc = np.array(g["k_cache"]), np.array(g["v_cache"])
    q = np.array(g["q"])[None]
    exp = np.array([[float(Fraction(x)) for x in row] for row in g["expected"]])
    out = paged_attention_decode(q, kc, vc, [g["block_table"]], [g["context_len"]], g["scale"],
                                 g["block_size"])
    assert np.allclose(out[0], exp, rtol=0, atol=1e-12)
    # same logits through doubled keys and scale 1/2
    out2 = paged_attention_decode(q, 2 * kc, vc, [g["block_table"]], [g["context_len"]], 0.5,
                                  g["block_size"])
    assert np.allclose(out2[0], exp, rtol=0, atol=1e-12)


def _random_problem(rng, B, hq, hkv, d, bs, nb, lens, dtype=np.float64):
    """Contiguous per-sequence K/V, then placed in a pool by a block manager
    with a random free order (the same path a serving step takes)."""
    bm = BlockManager(nb, bs, rng.permutation(nb))
    kc = np.full((nb, bs, hkv, d), np.nan)
    vc = np.full((nb, bs, hkv, d), np.nan)
    Ks, Vs = [], []
    for s, n in enumerate(lens):
        k = rng.standard_normal((n, hkv, d)).astype(dtype)
        v = rng.standard_normal((n, hkv, d)).astype(dtype)
        slots = bm.allocate(s, n)
        reshape_and_cache(k, v, kc, vc, np.array(slots, dtype=np.int64))
        Ks.append(k)
        Vs.append(v)
    mb = max(1, max(len(bm.block_table(s)) for s in range(B)))
    tables = np.zeros((B, mb), np.int64)
    for s in range(B):
        t = bm.block_table(s)
        tables[s, :len(t)] = t
    q = rng.standard_normal((B, hq, d))
    return q, kc, vc, tables, np.array(lens), Ks, Vs


def _sdpa_dense(q_s, K, V, scale):
    """torch fp64 SDPA over contiguous K/V; KV heads repeated for grouped queries."""
    hq, hkv = q_s.shape[0], K.shape[1]
    qt = torch.from_numpy(np.asarray(q_s, np.float64))[:, None, :]            # [Hq, 1, D]
    kt = torch.from_numpy(np.asarray(K, np.float64)).permute(1, 0, 2)          # [Hkv, n, D]
    vt = torch.from_numpy(np.asarray(V, np.float64)).permute(1, 0, 2)
    kt = kt.repeat_interleave(hq // hkv, dim=0)
    vt = vt.repeat_interleave(hq // hkv, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o[:, 0, :].numpy()


@pytest.mark.parametrize("hq,hkv,d,bs", [(4, 4, 16, 4), (8, 2, 32, 16), (6, 3, 8, 1), (8, 1, 64, 8)])
def test_matches_dense_sdpa(hq, hkv, d, bs):
    rng = np.random.default_rng(hq * 100 + hkv * 10 + d + bs)
    lens = [1, 2, bs - 1 if bs > 1 else 1, bs, bs + 1, 3 * bs + 5, 57]
    B = len(lens)
    nb = sum(-(-n // bs) for n in lens) + 7
    q, kc, vc, tables, ctx, Ks, Vs = _random_problem(rng, B, hq, hkv, d, bs, nb, lens)
    scale = 1.0 / math.sqrt(d)
    out = paged_attention_decode(q, kc, vc, tables, ctx, scale, bs)
    for s in range(B):
        ref = _sdpa_dense(q[s], Ks[s], Vs[s], scale)
        assert np.allclose(out[s], ref, rtol=0, atol=1e-12), s


def test_permutation_invariance_is_bitwise():
    rng = np.random.default_rng(7)
    bs, nb = 4, 40
    lens = [5, 17, 30]
    q, kc, vc, tables, ctx, _, _ = _random_problem(rng, 3, 4, 2, 8, bs, nb, lens)
    out = paged_attention_decode(q, kc, vc, tables, ctx, 0.3, bs)
    perm = rng.permutation(nb)                 # physical id b moves to perm[b]
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    out2 = paged_attention_decode(q, kc2, vc2, perm[tables], ctx, 0.3, bs)
    assert np.array_equal(out, out2)


def test_closed_forms():
    rng = np.random.default_rng(3)
    bs, d = 4, 8
    kc = rng.standard_normal((6, bs, 1, d))
    vc = rng.standard_normal((6, bs, 1, d))
    q = rng.standard_normal((1, 1, d))
    table = [[4, 2]]
    # one token: the output is that token's value, exactly
    out = paged_attention_decode(q, kc, vc, table, [1], 0.7, bs)
    assert np.array_equal(out[0, 0], vc[4, 0, 0])
    # two tokens: sigmoid-weighted mix
    x0, x1 = 0.7 * kc[4, 0, 0] @ q[0, 0], 0.7 * kc[4, 1, 0] @ q[0, 0]
    w = 1.0 / (1.0 + math.exp(x1 - x0))
    out = paged_attention_decode(q, kc, vc, table, [2], 0.7, bs)
    assert np.allclose(out[0, 0], w * vc[4, 0, 0] + (1 - w) * vc[4, 1, 0], atol=1e-14)
    # all keys equal: the mean of the values, across a block boundary
    kc_eq = np.broadcast_to(kc[0, 0], kc.shape).copy()
    out = paged_attention_decode(q, kc_eq, vc, table, [6], 0.7, bs)
    mean = np.concatenate([vc[4], vc[2, :2]])[:, 0].mean(axis=0)
    assert np.allclose(out[0, 0], mean, atol=1e-14)


def test_zero_context_gives_zeros():
    kc = np.full((2, 4, 1, 4), np.nan)
    out = paged_attention_decode(np.ones((1, 2, 4)), kc, kc, [[0]], [0], 1.0, 4)
    assert np.array_equal(out, np.zeros((1, 2, 4)))


def test_large_logits_are_stable():
    # softmax must not overflow for logits of a few hundred
    kc = np.zeros((1, 4, 1, 2))
    kc[0, :, 0, 0] = [100.0, 101.0, 99.0, 0.0]
    vc = np.zeros((1, 4, 1, 2))
    vc[0, :, 0, 1] = [1.0, 2.0, 3.0, 4.0]
    q = np.array([[[8.0, 0.0]]])
    out = paged_attention_decode(q, kc, vc, [[0]], [4], 1.0, 4)
    x = np.array([800.0, 808.0, 792.0, 0.0]) - 808.0
    p = np.exp(x)
    assert np.isfinite(out).all()
    assert np.allclose(out[0, 0, 1], (p @ [1, 2, 3, 4]) / p.sum(), atol=1e-14)
