"""The seeded input generators: determinism, shapes, ranges, bf16 rounding."""
import numpy as np
import pytest
import torch

from paged_kv_cache_322_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000, dtype=np.float32) * 10
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0]   # ties to even
    ours = wl.round_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(wl.bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_lengths_and_placement(name):
    w = wl.WORKLOADS[name]
    lens = wl.context_lens(w)
    assert lens.shape == (w.num_seqs,)
    assert np.array_equal(lens, wl.context_lens(w))
    if w.ctx == "fixed":
        assert tuple(lens) == w.fixed
    elif w.ctx == "shared_prefix":
        assert lens.min() >= w.shared_prefix + w.lo and lens.max() <= w.shared_prefix + w.hi
    else:
        assert lens.min() >= w.lo and lens.max() <= w.hi
    order = wl.free_order(w)
    assert np.array_equal(np.sort(order), np.arange(w.num_blocks))
    need = sum(-(-int(n) // w.block_size) for n in lens)
    assert need < w.num_blocks


def test_per_sequence_streams_are_independent_of_batch():
    w = wl.WORKLOADS["tiny_fp32"]
    lens = wl.context_lens(w)
    allkv = wl.prompt_kv_all(w, lens, threads=2)
    k2, v2 = wl.prompt_kv(w, 2, int(lens[2]))
    assert np.array_equal(allkv[2][0], k2) and np.array_equal(allkv[2][1], v2)
    assert k2.dtype == np.float32 and k2.shape == (lens[2], w.num_kv_heads, w.head_dim)


def test_shared_prefix_is_shared():
    w = wl.WORKLOADS["shared_prefix"]
    lens = wl.context_lens(w)
    k0, _ = wl.prompt_kv(w, 0, int(lens[0]))
    k5, _ = wl.prompt_kv(w, 5, int(lens[5]))
    p = w.shared_prefix
    assert np.array_equal(k0[:p], k5[:p]) and not np.array_equal(k0[p:p + 8], k5[p:p + 8])


def test_bf16_values_are_representable():
    w = wl.WORKLOADS["llama2_7b"]
    q = wl.decode_q(w, 0)
    assert np.array_equal(wl.bf16_bits_to_f32(wl.round_to_bf16(q)), q)
