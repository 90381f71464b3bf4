"""Pins of the oracle's causal multi-query paged attention (CPU only):
a whole prompt attended at once equals torch's causal scaled-dot-product
attention on the contiguous sequence (an independent library routine); a
prompt fed in chunks gives the same rows; all-equal keys give the running mean
of the visible values (so the causal window is exactly 0..position); one query
per sequence is the decode oracle; physical placement does not matter."""
import math

import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager

BS = 4


def _cache(lens, hkv, d, rng, nb=None, order=None):
    nb = nb or sum(-(-n // BS) for n in lens) + 5
    bm = BlockManager(nb, BS, order if order is not None else rng.permutation(nb))
    kc = np.full((nb, BS, hkv, d), np.nan)
    vc = np.full((nb, BS, hkv, d), np.nan)
    data = []
    for s, n in enumerate(lens):
        k = rng.standard_normal((n, hkv, d))
        v = rng.standard_normal((n, hkv, d))
        ocache.reshape_and_cache(k, v, kc, vc, np.asarray(bm.allocate(s, n)))
        data.append((k, v))
    return bm, kc, vc, data


def _sdpa_causal(q, k, v, scale):
    """q [n, Hq, D], k/v [n, Hkv, D]: torch causal SDPA in fp64 (heads repeated for GQA)."""
    g = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q).double().permute(1, 0, 2)
    kt = torch.from_numpy(k).double().repeat_interleave(g, dim=1).permute(1, 0, 2)
    vt = torch.from_numpy(v).double().repeat_interleave(g, dim=1).permute(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (6, 3)])
def test_whole_prompt_equals_causal_sdpa(hq, hkv):
    rng = np.random.default_rng(hq * 10 + hkv)
    lens = [1, 7, 12, 30]
    d = 8
    bm, kc, vc, data = _cache(lens, hkv, d, rng)
    qs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), hq, d))
    scale = 1 / math.sqrt(d)
    out = oattn.paged_attention_multi_query(q, kc, vc, [bm.block_table(s) for s in range(len(lens))], lens, qs,
                                            scale, BS)
    for s, n in enumerate(lens):
        exp = _sdpa_causal(q[qs[s]:qs[s + 1]], data[s][0], data[s][1], scale)
        np.testing.assert_allclose(out[qs[s]:qs[s + 1]], exp, rtol=0, atol=1e-12)


def test_chunks_give_the_rows_of_the_whole_prompt():
    """A 23-token prompt as chunks of 5, 1, 9, 8 tokens: each chunk attends with
    context = tokens so far; the rows match one whole-prompt pass."""
    rng = np.random.default_rng(3)
    hq, hkv, d, L = 4, 2, 8, 23
    bm, kc, vc, data = _cache([L], hkv, d, rng)
    q = rng.standard_normal((L, hq, d))
    table = [bm.block_table(0)]
    whole = oattn.paged_attention_multi_query(q, kc, vc, table, [L], np.array([0, L]), 0.3, BS)
    done = 0
    for c in (5, 1, 9, 8):
        part = oattn.paged_attention_multi_query(q[done:done + c], kc, vc, table, [done + c], np.array([0, c]), 0.3, BS)
        np.testing.assert_allclose(part, whole[done:done + c], rtol=0, atol=1e-12)
        done += c
    assert done == L


def test_equal_keys_give_running_mean_of_values():
    rng = np.random.default_rng(4)
    hkv, d = 2, 5
    lens = [9, 14]
    bm, kc, vc, data = _cache(lens, hkv, d, rng)
    kc[...] = 0.7                                   # every key the same -> uniform weights
    n = [3, 14]                                     # spec-verify-like tail of 3, and a whole prompt
    qs = np.array([0, 3, 17], dtype=np.int32)
    q = rng.standard_normal((17, hkv * 2, d))
    out = oattn.paged_attention_multi_query(q, kc, vc, [bm.block_table(s) for s in range(2)], lens, qs, 1.0, BS)
    for s in range(2):
        v = data[s][1]
        for i in range(n[s]):
            p = lens[s] - n[s] + i
            exp = v[:p + 1].mean(axis=0)            # [Hkv, D]
            got = out[qs[s] + i].reshape(hkv, 2, d)
            for h in range(2):
                np.testing.assert_allclose(got[:, h], exp, rtol=0, atol=1e-12)


def test_one_query_per_sequence_is_decode():
    rng = np.random.default_rng(5)
    lens = [1, 16, 33]
    bm, kc, vc, _ = _cache(lens, 2, 8, rng)
    tables = [bm.block_table(s) for s in range(3)]
    q = rng.standard_normal((3, 4, 8))
    mq = oattn.paged_attention_multi_query(q, kc, vc, tables, lens, np.arange(4), 0.35, BS)
    dec = oattn.paged_attention_decode(q, kc, vc, tables, lens, 0.35, BS)
    np.testing.assert_array_equal(mq, dec)


def test_brute_force_tiny():
    """Two sequences, D = 2, written out with Python floats and math.exp."""
    rng = np.random.default_rng(6)
    lens, n = [6, 3], [2, 3]
    bm, kc, vc, data = _cache(lens, 1, 2, rng)
    qs = np.array([0, 2, 5], dtype=np.int32)
    q = rng.standard_normal((5, 2, 2))
    out = oattn.paged_attention_multi_query(q, kc, vc, [bm.block_table(s) for s in range(2)], lens, qs, 0.5, BS)
    for s in range(2):
        k, v = data[s]
        for i in range(n[s]):
            pos = lens[s] - n[s] + i
            for h in range(2):
                x = [0.5 * sum(float(q[qs[s] + i, h, c]) * float(k[j, 0, c]) for c in range(2)) for j in range(pos + 1)]
                mx = max(x)
                w = [math.exp(t - mx) for t in x]
                for c in range(2):
                    exp = sum(w[j] * float(v[j, 0, c]) for j in range(pos + 1)) / sum(w)
                    assert abs(out[qs[s] + i, h, c] - exp) < 1e-12


def test_physical_placement_does_not_matter():
    rng = np.random.default_rng(7)
    lens = [10, 21]
    qs = np.array([0, 4, 11], dtype=np.int32)
    res = []
    for order_seed in (1, 2):
        r = np.random.default_rng(99)
        nb = 20
        bm, kc, vc, _ = _cache(lens, 2, 4, r, nb=nb, order=np.random.default_rng(order_seed).permutation(nb))
        q = np.random.default_rng(100).standard_normal((11, 4, 4))
        res.append(oattn.paged_attention_multi_query(q, kc, vc, [bm.block_table(s) for s in range(2)], lens, qs,
                                                     0.4, BS))
    np.testing.assert_array_equal(res[0], res[1])


def test_more_queries_than_context_is_refused():
    with pytest.raises(ValueError):
        oattn.paged_attention_multi_query(np.zeros((3, 1, 2)), np.zeros((2, BS, 1, 2)), np.zeros((2, BS, 1, 2)),
                                          [[0]], [2], np.array([0, 3]), 1.0, BS)
