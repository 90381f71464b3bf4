"""GPU parity of the paged path at block sizes 8, 32 and 64 ("vLLM
PagedAttention 深度解析" §8.1: block sizes are powers of two, 16 the default;
smaller blocks waste less, larger ones stream longer runs). Every consumer path
(SIMT fp32 / bf16 MHA, tensor-core GQA, FP8 SIMT and tensor-core) against the
fp64 oracle at ragged contexts around block, stage and partition boundaries;
the native decode step; and the bitwise invariance of the result under a
permutation of physical blocks."""
import dataclasses

import numpy as np
import pytest
import torch

from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem, step_inputs, tolerance
from tests.test_gpu_attention import _edge_problem, _run
from tests.test_gpu_fp8 import fp8_edge_case

pytestmark = pytest.mark.gpu

BLOCK_SIZES = [8, 32, 64]
LENS = [0, 1, 7, 8, 9, 15, 16, 17, 31, 32, 33, 63, 64, 65, 200, 511, 513, 1000]


@pytest.mark.parametrize("bs", BLOCK_SIZES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("hq,hkv,d", [(4, 4, 128), (8, 2, 128), (16, 2, 64), (8, 8, 64)])
@pytest.mark.parametrize("part", [0, 64, 256])
def test_block_size_edge_contexts(bs, dtype, hq, hkv, d, part):
    dev, ref = _edge_problem(bs * 7 + hq + d, hq, hkv, d, dtype, LENS, bs=bs)
    out = _run(dev, partition_tokens=part)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.array_equal(got[0], np.zeros_like(got[0]))
    assert np.abs(got - ref).max() <= (1e-5 if dtype == "f32" else 2e-3)


@pytest.mark.parametrize("bs", BLOCK_SIZES)
@pytest.mark.parametrize("hq,hkv", [(4, 4), (16, 4), (16, 2)])
@pytest.mark.parametrize("part", [0, 64])
def test_block_size_fp8_edge_contexts(bs, hq, hkv, part):
    fp8_edge_case(hq, hkv, part, bs=bs)


@pytest.mark.parametrize("bs", BLOCK_SIZES)
def test_block_size_permutation_invariance(bs):
    dev, _ = _edge_problem(11 + bs, 32, 8, 128, "bf16", [700, 33, 1024], bs=bs)
    out1 = _run(dev, partition_tokens=256)
    nb = dev["nb"]
    perm = torch.from_numpy(np.random.default_rng(bs).permutation(nb)).cuda()
    kc2, vc2 = torch.empty_like(dev["kc"]), torch.empty_like(dev["vc"])
    kc2[perm], vc2[perm] = dev["kc"], dev["vc"]
    out2 = _run(dict(dev, kc=kc2, vc=vc2, tables=perm[dev["tables"].long()].int().contiguous()),
                partition_tokens=256)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("bs", BLOCK_SIZES)
@pytest.mark.parametrize("name", ["llama2_7b", "gqa_70b", "gqa_70b_fp8"])
def test_block_size_decode_steps(bs, name):
    """Prompts, two decode steps (append + attention) through the engine, and
    one step through the native C step, at block size bs."""
    base = wl.WORKLOADS[name]
    w = dataclasses.replace(base, block_size=bs, num_seqs=5, num_blocks=base.num_blocks * 16 // bs // 8)
    cache, lens = gpu_problem(w)
    op = OracleProblem(w)
    for step in range(2):
        q, kn, vn = step_inputs(w, step)
        out = cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale)
        ref = op.decode_step(step)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert np.abs(out.cpu().numpy().astype(np.float64) - ref).max() <= tolerance(w)
    # the native step from host buffers
    dt = torch.bfloat16 if w.kv_dtype != "f32" else torch.float32
    step = binding.DecodeStep(cache.bm, cache.k_cache, cache.v_cache, max_seqs=w.num_seqs,
                              num_q_heads=w.num_q_heads, max_blocks_per_seq=cache.max_blocks_per_seq,
                              out_dtype=torch.float32, kv_scales=(w.kv_scale, w.kv_scale))
    q, kn, vn = (torch.from_numpy(x).to(dt).pin_memory() for x in (wl.decode_q(w, 2), *wl.decode_kv(w, 2)))
    out_h = torch.empty((w.num_seqs, w.num_q_heads, w.head_dim), dtype=torch.float32).pin_memory()
    step(np.arange(w.num_seqs), q, kn, vn, out_h, w.scale)
    torch.cuda.synchronize()
    ref = op.decode_step(2)
    assert binding.get_device_error() == 0
    assert np.abs(out_h.numpy().astype(np.float64) - ref).max() <= tolerance(w)
