"""GPU parity of the FP8 (e4m3) KV cache: the quantising append is bit-exact
against the oracle's encoder, and attention over the FP8 cache matches the
oracle's fp64 attention over the same dequantised values (<= 2e-3)."""
import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from oracle import fp8 as ofp8
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem, step_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("in_dtype,scale", [(torch.bfloat16, 1 / 64), (torch.float32, 0.0123), (torch.float32, 1.0)])
def test_quantising_append_is_bit_exact(in_dtype, scale):
    rng = np.random.default_rng(5)
    nb, bs, hkv, d, T = 32, 16, 4, 128, 40
    x = rng.standard_normal((2, T, hkv, d)).astype(np.float32) * 9
    # exact ties between neighbouring codes, saturation, zeros and tiny values
    codes = np.arange(256)
    vals = ofp8.decode_array(codes)
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = ((fin[1:] + fin[:-1]) / 2).astype(np.float32)
    x[0, 0].flat[:mids.size] = mids * np.float32(scale) if in_dtype == torch.float32 else mids[0]
    x[0, 1].flat[:8] = [500, -500, 1e9, -1e9, 0.0, -0.0, 1e-12, 448.0]
    x[1, 0].flat[:8] = [v * scale for v in (500, -500, 1e9, -1e9, 0.0, -0.0, 1e-12, 448.0)]
    if in_dtype == torch.bfloat16:
        x = wl.bf16_bits_to_f32(wl.round_to_bf16(x))
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[3] = -1
    kc = torch.full((nb, bs, hkv, d), 0x7F, dtype=torch.uint8, device="cuda")
    vc = kc.clone()
    k = torch.from_numpy(x[0]).cuda().to(in_dtype)
    v = torch.from_numpy(x[1]).cuda().to(in_dtype)
    binding.reshape_and_cache_fp8(k, v, kc, vc, torch.from_numpy(slots).cuda(), scale, scale)
    ko = np.full((nb, bs, hkv, d), 0x7F, np.uint8)
    vo = ko.copy()
    ocache.reshape_and_cache_fp8(x[0], x[1], ko, vo, slots, scale, scale)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.array_equal(kc.cpu().numpy(), ko) and np.array_equal(vc.cpu().numpy(), vo)


SMALL = {
    "llama2_7b_fp8": dataclasses.replace(wl.WORKLOADS["llama2_7b_fp8"], num_seqs=6, num_blocks=2048),
    "gqa_70b_fp8": dataclasses.replace(wl.WORKLOADS["gqa_70b_fp8"], num_seqs=5, num_blocks=4096),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("part", [0, 512])
def test_fp8_decode_steps_match_oracle(name, part):
    w = SMALL[name]
    cache, lens = gpu_problem(w)
    op = OracleProblem(w)
    for step in range(2):
        q, kn, vn = step_inputs(w, step)
        out = cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale, partition_tokens=part)
        ref = op.decode_step(step)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3


EDGE = [1, 2, 15, 16, 17, 33, 255, 513, 1000]


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (16, 4), (16, 2), (32, 2), (16, 1)])
@pytest.mark.parametrize("part", [0, 64])
def test_fp8_edge_contexts(hq, hkv, part):
    """(32, 2) and (16, 1): group 16, two 8-wide head tiles (two KV heads per CTA, and one)."""
    fp8_edge_case(hq, hkv, part)


def fp8_edge_case(hq, hkv, part, bs=16):
    """Ragged contexts through the FP8 append and attention, against the oracle."""
    rng = np.random.default_rng(hq * 10 + hkv + bs)
    d, scale = 128, 1 / 32
    nb = sum(-(-n // bs) for n in EDGE) + 9
    order = rng.permutation(nb).astype(np.int32)
    mb = max(-(-n // bs) for n in EDGE)
    kc = torch.full((nb, bs, hkv, d), 0x7F, dtype=torch.uint8, device="cuda")
    vc = kc.clone()
    ko = np.full((nb, bs, hkv, d), 0x7F, np.uint8)
    vo = ko.copy()
    pbm, obm = binding.BlockManager(nb, bs, order), OracleBM(nb, bs, order)
    for s, n in enumerate(EDGE):
        k = wl.bf16_bits_to_f32(wl.round_to_bf16(rng.standard_normal((n, hkv, d)).astype(np.float32)))
        v = wl.bf16_bits_to_f32(wl.round_to_bf16(rng.standard_normal((n, hkv, d)).astype(np.float32)))
        ps = pbm.allocate(s, n)
        assert ps.tolist() == obm.allocate(s, n)
        binding.reshape_and_cache_fp8(torch.from_numpy(k).cuda().bfloat16(), torch.from_numpy(v).cuda().bfloat16(),
                                      kc, vc, torch.from_numpy(ps).cuda(), scale, scale)
        ocache.reshape_and_cache_fp8(k, v, ko, vo, ps, scale, scale)
    tables, plens = pbm.block_tables(np.arange(len(EDGE)), mb)
    q = wl.bf16_bits_to_f32(wl.round_to_bf16(rng.standard_normal((len(EDGE), hq, d)).astype(np.float32)))
    out = torch.empty((len(EDGE), hq, d), dtype=torch.float32, device="cuda")
    binding.paged_attention_decode_fp8(out, torch.from_numpy(q).cuda().bfloat16(), kc, vc,
                                       torch.from_numpy(tables).cuda(), torch.from_numpy(plens).cuda(),
                                       1 / math.sqrt(d), scale, scale, partition_tokens=part)
    ref = oattn.paged_attention_decode_fp8(q, ko, vo, [obm.block_table(s) for s in range(len(EDGE))], EDGE,
                                           1 / math.sqrt(d), bs, scale, scale)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3


def test_fp8_persistent_schedule_is_refused():
    kc = torch.zeros((4, 16, 2, 128), dtype=torch.uint8, device="cuda")
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, 4, 128), device="cuda")
    t = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(binding.PkvError) as e:
        binding.paged_attention_decode_fp8(out, q, kc, kc, t, t[0], 0.1, 1.0, 1.0, partition_tokens=-1)
    assert e.value.status == 2


@pytest.mark.parametrize("name", ["llama2_7b_fp8", "gqa_70b_fp8"])
def test_fp8_full_size_sampled(name):
    w = wl.WORKLOADS[name]
    sample = wl.sample_seqs(w, 6)
    cache, lens = gpu_problem(w, fill_nan=False)
    op = OracleProblem(w, keep=sample)
    q, kn, vn = step_inputs(w, 0)
    out = cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale)
    ref = op.decode_step(0, seqs=sample)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got[sample].astype(np.float64) - ref).max() <= 2e-3
