"""GPU parity of the shared-prefix decode (a cascade that reads a batch's shared
prefix blocks once) against the fp64 oracle's plain decode attention over each
sequence's whole context ("为什么PagedAttention能让大模型推理吞吐量提升数倍",
Memory Sharing: sequences forked from one prompt map the same physical blocks).
Block tables are built here from a seeded permutation: the prefix blocks first
in every row, then each sequence's own tail blocks."""
import math

import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.test_gpu_attention import check_bf16_out

pytestmark = pytest.mark.gpu


def _bf16(x):
    return wl.bf16_bits_to_f32(wl.round_to_bf16(np.asarray(x, np.float32)))


def _problem(seed, B, hq, hkv, bs, prefix_blocks, tails, d=128):
    rng = np.random.default_rng(seed)
    P = prefix_blocks * bs
    own = [-(-t // bs) for t in tails]
    nb = prefix_blocks + sum(own) + 9
    order = rng.permutation(nb).astype(np.int32)
    prefix_ids = order[:prefix_blocks]
    mb = prefix_blocks + max(own)
    tables = np.zeros((B, mb), np.int32)
    kc = torch.full((nb, bs, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    ko = np.full((nb, bs, hkv, d), np.nan, np.float32)
    vo = ko.copy()

    def put(k, v, ids):
        slots = np.array([int(ids[j // bs]) * bs + j % bs for j in range(k.shape[0])], np.int64)
        binding.reshape_and_cache(torch.from_numpy(k).cuda().bfloat16(), torch.from_numpy(v).cuda().bfloat16(),
                                  kc, vc, torch.from_numpy(slots).cuda())
        ocache.reshape_and_cache(k, v, ko, vo, slots)

    put(_bf16(rng.standard_normal((P, hkv, d))), _bf16(rng.standard_normal((P, hkv, d))), prefix_ids)
    at = prefix_blocks
    for s, t in enumerate(tails):
        ids = order[at:at + own[s]]
        at += own[s]
        tables[s, :prefix_blocks] = prefix_ids
        tables[s, prefix_blocks:prefix_blocks + own[s]] = ids
        put(_bf16(rng.standard_normal((t, hkv, d))), _bf16(rng.standard_normal((t, hkv, d))), ids)
    lens = np.array([P + t for t in tails], np.int32)
    q = _bf16(rng.standard_normal((B, hq, d)))
    scale = 1 / math.sqrt(d)
    ref = oattn.paged_attention_decode(q, ko, vo, tables, lens, scale, bs)
    dev = dict(q=torch.from_numpy(q).cuda().bfloat16(), kc=kc, vc=vc, tables=torch.from_numpy(tables).cuda(),
               lens=torch.from_numpy(lens).cuda(), scale=scale, prefix=P, maxlen=int(lens.max()))
    return dev, ref


def _cascade(dev, out_dtype=torch.float32):
    out = torch.empty(dev["q"].shape, dtype=out_dtype, device="cuda")
    binding.paged_attention_decode_shared_prefix(out, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"],
                                                 dev["prefix"], dev["scale"], dev["maxlen"])
    return out


@pytest.mark.parametrize("B,hq,hkv", [(32, 32, 32), (8, 64, 8), (40, 8, 8), (4, 128, 8), (16, 32, 16)])
@pytest.mark.parametrize("bs", [8, 16, 32, 64])
def test_shared_prefix_matches_oracle(B, hq, hkv, bs):
    """Prefix of several blocks (crossing the 128-token tiles), tails from 1 token
    (the sequence's own new token only) up to several blocks, ragged."""
    rng = np.random.default_rng(B * 1000 + bs)
    tails = [1, bs, bs + 1] + rng.integers(1, 300, size=B - 3).tolist()
    dev, ref = _problem(7 + B + bs, B, hq, hkv, bs, max(1, 320 // bs), tails)
    out = _cascade(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - ref).max() <= 2e-3
    check_bf16_out(_cascade(dev, torch.bfloat16), ref)


def test_shared_prefix_config4_shape_matches_plain_decode():
    """The shared-prefix workload's shape (32 sequences, 32/32 heads, a 1008-token
    shared prefix of 63 blocks, tails 64-512): the cascade and the regular decode
    call both within 2e-3 of the oracle."""
    rng = np.random.default_rng(404)
    tails = rng.integers(64, 513, size=32).tolist()
    dev, ref = _problem(404, 32, 32, 32, 16, 63, tails)
    out = _cascade(dev)
    plain = torch.empty_like(out)
    binding.paged_attention_decode(plain, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"], dev["scale"],
                                   max_context_len=dev["maxlen"])
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3
    assert np.abs(plain.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3


def test_shared_prefix_context_not_past_prefix_is_flagged():
    """A context that does not reach past the prefix breaks the call's contract:
    flagged PKV_ERR_DEVICE_BOUNDS in the device word, the launch completes."""
    dev, _ = _problem(9, 32, 32, 32, 16, 4, [5] * 32)
    dev["lens"][3] = dev["prefix"]
    _cascade(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 4


def test_shared_prefix_refusals():
    """Host-side refusals before any launch: too few query rows per KV head for
    the tcgen05 prefix kernel, a prefix that is not whole blocks."""
    dev, _ = _problem(10, 8, 8, 8, 16, 2, [3] * 8)               # 8 sequences x group 1 = 8 rows
    with pytest.raises(binding.PkvError):
        _cascade(dev)
    dev, _ = _problem(11, 32, 32, 32, 16, 2, [3] * 32)
    dev["prefix"] = 20
    with pytest.raises(binding.PkvError):
        _cascade(dev)


def test_shared_prefix_long_prefix_fewer_partitions_than_sized():
    """A 4000-token prefix over 16 KV heads: the workspace is sized for 9 prefix
    partitions (one wave of 148 CTAs), whole 512-token ones give 8 (the last one
    ragged)."""
    rng = np.random.default_rng(77)
    tails = rng.integers(1, 200, size=16).tolist()
    dev, ref = _problem(77, 16, 32, 16, 16, 250, tails)
    out = _cascade(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3


def test_shared_prefix_tail_cap_past_unit_bins_takes_grid_order():
    """max_context_len 70000 tokens past a 512-token prefix: a tail partition of
    more than 4096 blocks has no longest-first list, the tails run in grid order."""
    rng = np.random.default_rng(78)
    tails = rng.integers(1, 400, size=32).tolist()
    dev, ref = _problem(78, 32, 32, 32, 16, 32, tails)
    maxlen = 512 + 70000
    t = dev["tables"]
    wide = torch.zeros((t.shape[0], -(-maxlen // 16)), dtype=torch.int32, device="cuda")
    wide[:, :t.shape[1]] = t
    dev["tables"], dev["maxlen"] = wide, maxlen
    out = _cascade(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3
