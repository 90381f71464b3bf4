"""The pins catch plausible mistakes: each test plants one mistake in a copy of
an oracle function (on the CPU) and checks that a pin from
test_oracle_attention / test_oracle_cache_ops now fails."""
import math

import numpy as np
import pytest

import oracle.paged_attention as pa
from oracle.block_manager import BlockManager
from tests.test_oracle_attention import _random_problem, _sdpa_dense


def _dense_pin_holds(attend_fn, gather_fn, hq=8, hkv=2, d=16, bs=4):
    rng = np.random.default_rng(11)
    lens = [1, 3, 4, 5, 13]
    nb = 20
    q, kc, vc, tables, ctx, Ks, Vs = _random_problem(rng, len(lens), hq, hkv, d, bs, nb, lens)
    scale = 1.0 / math.sqrt(d)
    for s in range(len(lens)):
        K = gather_fn(kc, tables[s], int(ctx[s]), bs)
        V = gather_fn(vc, tables[s], int(ctx[s]), bs)
        out = attend_fn(q[s], K, V, scale)
        if not np.allclose(out, _sdpa_dense(q[s], Ks[s], Vs[s], scale), atol=1e-10, equal_nan=False):
            return False
    return True


def test_unmodified_oracle_passes():
    assert _dense_pin_holds(pa.attend, pa.gather_logical)


def _attend_wrong_group(q_s, K, V, scale):
    hq, hkv = q_s.shape[0], K.shape[1]
    out = np.zeros((hq, q_s.shape[1]))
    for h in range(hq):
        g = h % hkv                                  # mistake: interleaved groups
        x = scale * (K[:, g, :] @ q_s[h])
        p = np.exp(x - x.max())
        out[h] = (p @ V[:, g, :]) / p.sum()
    return out


def _attend_no_scale(q_s, K, V, scale):
    return pa.attend(q_s, K, V, 1.0)                 # mistake: scale dropped


def _attend_no_normalise(q_s, K, V, scale):
    hq, hkv = q_s.shape[0], K.shape[1]
    out = np.zeros((hq, q_s.shape[1]))
    for h in range(hq):
        g = h // (hq // hkv)
        x = scale * (K[:, g, :] @ q_s[h])
        out[h] = np.exp(x - x.max()) @ V[:, g, :]   # mistake: missing / sum
    return out


def _attend_k_for_v(q_s, K, V, scale):
    return pa.attend(q_s, K, K, scale)               # mistake: keys used as values


def _gather_offset_major(cache, row, ctx, bs):
    n_blk = -(-ctx // bs)
    blocks = np.asarray(cache[np.asarray(row[:n_blk])], np.float64)
    flat = blocks.transpose(1, 0, 2, 3).reshape((n_blk * bs,) + blocks.shape[2:])
    return flat[:ctx]                                # mistake: offset-major order


def _gather_drop_last(cache, row, ctx, bs):
    return pa.gather_logical(cache, row, ctx, bs)[:max(ctx - 1, 1)]   # mistake: off by one


def _gather_identity_table(cache, row, ctx, bs):
    n_blk = -(-ctx // bs)
    return pa.gather_logical(cache, list(range(n_blk)), ctx, bs)       # mistake: table ignored


@pytest.mark.parametrize("attend_fn,gather_fn", [
    (_attend_wrong_group, pa.gather_logical),
    (_attend_no_scale, pa.gather_logical),
    (_attend_no_normalise, pa.gather_logical),
    (_attend_k_for_v, pa.gather_logical),
    (pa.attend, _gather_offset_major),
    (pa.attend, _gather_drop_last),
    (pa.attend, _gather_identity_table),
])
def test_planted_mistake_is_caught(attend_fn, gather_fn):
    assert not _dense_pin_holds(attend_fn, gather_fn)


def test_planted_allocator_mistake_is_caught():
    """A block manager that forgets copy-on-write breaks the page's CoW example."""
    class NoCow(BlockManager):
        def append_slot(self, seq):
            n = self.lens[seq]
            if n % self.block_size != 0:
                self.lens[seq] = n + 1
                return self.slot(seq, n), None
            return super().append_slot(seq)

    bm = NoCow(8, 4, [7, 1, 3, 0, 2, 4, 5, 6])
    bm.allocate("A1", 7)
    bm.fork("A1", "A2")
    slot, copy = bm.append_slot("A1")
    assert (slot, copy) != (15, (1, 3))
