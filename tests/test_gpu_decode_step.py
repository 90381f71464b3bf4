"""The native decode step (pkv_decode_step, host buffers in and out) against
the same step sequenced call by call from Python, and against the oracle."""
import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from oracle import paged_attention as oattn
from oracle.block_manager import BlockManager as OracleBM
from paged_kv_cache_322_b200 import binding, workloads as wl
from paged_kv_cache_322_b200.engine import PagedKVCache

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pinned_out", [True, False])
@pytest.mark.parametrize("hq,hkv,part", [(32, 8, 0), (16, 16, -1), (8, 2, 64)])
def test_native_step_matches_python_step_and_oracle(hq, hkv, part, pinned_out):
    """pinned_out: the output buffer is page-locked (the kernels write it through
    its device mapping) or pageable (a copy after the kernels)."""
    rng = np.random.default_rng(hq + hkv)
    nb, bs, d, mb = 256, 16, 128, 64
    order = rng.permutation(nb).astype(np.int32)
    lens = [33, 100, 7, 250, 16]

    def bf(*shape):
        return wl.bf16_bits_to_f32(wl.round_to_bf16(rng.standard_normal(shape, dtype=np.float32)))

    prompts = [(bf(n, hkv, d), bf(n, hkv, d)) for n in lens]
    caches = []
    for _ in range(2):
        c = PagedKVCache(nb, bs, hkv, d, torch.bfloat16, "cuda", free_order=order, max_blocks_per_seq=mb,
                         fill_value=float("nan"))
        for s, (k, v) in enumerate(prompts):
            c.add_sequence(s, torch.from_numpy(k).cuda().bfloat16(), torch.from_numpy(v).cuda().bfloat16())
        c.fork(1, 5)               # sequence 5 shares 1's blocks: its first append copies the partial block
        c.fork(3, 6)
        caches.append(c)
    obm = OracleBM(nb, bs, order)
    ko = np.full((nb, bs, hkv, d), np.nan, np.float32)
    vo = np.full_like(ko, np.nan)
    for s, (k, v) in enumerate(prompts):
        ocache.reshape_and_cache(k, v, ko, vo, np.asarray(obm.allocate(s, len(k))))
    obm.fork(1, 5)
    obm.fork(3, 6)
    ids = np.array([0, 1, 2, 3, 4, 5, 6], dtype=np.int64)
    step = binding.DecodeStep(caches[1].bm, caches[1].k_cache, caches[1].v_cache, max_seqs=8, num_q_heads=hq,
                              max_blocks_per_seq=mb, out_dtype=torch.float32, partition_tokens=part)
    scale = 1.0 / np.sqrt(d)
    for it in range(3):
        q, kn, vn = bf(len(ids), hq, d), bf(len(ids), hkv, d), bf(len(ids), hkv, d)
        qh = torch.from_numpy(q).bfloat16().pin_memory()
        kh = torch.from_numpy(kn).bfloat16().pin_memory()
        vh = torch.from_numpy(vn).bfloat16().pin_memory()
        out_py = caches[0].decode_step(ids, qh.cuda(), kh.cuda(), vh.cuda(), scale, partition_tokens=part)
        out_host = torch.empty((len(ids), hq, d), dtype=torch.float32)
        if pinned_out:
            out_host = out_host.pin_memory()
        step(ids, qh, kh, vh, out_host, scale)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert torch.equal(out_py.cpu(), out_host)                     # same kernels, same inputs
        slots, pairs = [], []
        for s in ids:
            slot, cp = obm.append_slot(int(s))
            slots.append(slot)
            if cp:
                pairs.append(cp)
        assert len(pairs) == (2 if it == 0 else 0)
        if pairs:
            ocache.copy_blocks(ko, vo, [a for a, _ in pairs], [b for _, b in pairs])
        ocache.reshape_and_cache(kn, vn, ko, vo, np.asarray(slots))
        ref = oattn.paged_attention_decode(q, ko, vo, [obm.block_table(int(s)) for s in ids],
                                           [obm.lens[int(s)] for s in ids], scale, bs)
        assert np.abs(out_host.numpy() - ref).max() <= 2e-3
    for a, b in ((caches[0].k_cache, caches[1].k_cache), (caches[0].v_cache, caches[1].v_cache)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_native_step_phase_timing():
    """The context's phase timing: every phase measured, the output unchanged."""
    rng = np.random.default_rng(11)
    nb, bs, hq, hkv, d, mb = 128, 16, 16, 4, 128, 32
    c = PagedKVCache(nb, bs, hkv, d, torch.bfloat16, "cuda", free_order=rng.permutation(nb).astype(np.int32),
                     max_blocks_per_seq=mb)
    for s, n in enumerate([40, 300, 17]):
        k = torch.randn((n, hkv, d), device="cuda").bfloat16()
        c.add_sequence(s, k, k.clone())
    step = binding.DecodeStep(c.bm, c.k_cache, c.v_cache, max_seqs=4, num_q_heads=hq, max_blocks_per_seq=mb,
                              out_dtype=torch.float32)
    ids = np.arange(3, dtype=np.int64)
    with pytest.raises(binding.PkvError):
        step.last_timing()                       # nothing timed yet
    step.set_timing(True)
    qh = torch.randn((3, hq, d)).bfloat16().pin_memory()
    kh = torch.randn((3, hkv, d)).bfloat16().pin_memory()
    out_host = torch.empty((3, hq, d), dtype=torch.float32).pin_memory()
    step(ids, qh, kh, kh.clone(), out_host, 0.1)
    t = step.last_timing()
    assert binding.get_device_error() == 0
    assert set(t) == {"host_block_manager", "h2d", "kernels", "d2h"}
    assert all(v >= 0 for v in t.values()) and t["kernels"] > 0
    assert torch.isfinite(out_host).all()
    step.set_timing(False)


def test_native_steps_in_flight_together():
    """Steps issued back to back, each result read only after the next step was
    issued (the pipelined use): every output equals the one of the same steps run
    one at a time on a twin cache."""
    rng = np.random.default_rng(12)
    nb, bs, hq, hkv, d, mb = 256, 16, 16, 4, 128, 64
    order = rng.permutation(nb).astype(np.int32)
    lens = [100, 33, 500, 7]
    prompts = [(torch.randn((n, hkv, d), device="cuda").bfloat16(), torch.randn((n, hkv, d), device="cuda").bfloat16())
               for n in lens]
    caches, steps = [], []
    for _ in range(2):
        c = PagedKVCache(nb, bs, hkv, d, torch.bfloat16, "cuda", free_order=order, max_blocks_per_seq=mb)
        for s_, (k, v) in enumerate(prompts):
            c.add_sequence(s_, k, v)
        caches.append(c)
        steps.append(binding.DecodeStep(c.bm, c.k_cache, c.v_cache, max_seqs=4, num_q_heads=hq, max_blocks_per_seq=mb,
                                        out_dtype=torch.float32))
    ids = np.arange(4, dtype=np.int64)
    inputs = [tuple(torch.randn(shape).bfloat16().pin_memory() for shape in ((4, hq, d), (4, hkv, d), (4, hkv, d)))
              for _ in range(6)]
    serial = []
    for q, k, v in inputs:
        o = torch.empty((4, hq, d), dtype=torch.float32).pin_memory()
        steps[0](ids, q, k, v, o, 0.1)
        torch.cuda.current_stream().synchronize()
        serial.append(o.clone())
    outs = [torch.empty((4, hq, d), dtype=torch.float32).pin_memory() for _ in inputs]
    evs = []
    for j, (q, k, v) in enumerate(inputs):
        steps[1](ids, q, k, v, outs[j], 0.1)
        e = torch.cuda.Event()
        e.record()
        evs.append(e)
        if j >= 1:
            evs[j - 1].synchronize()
            assert torch.equal(outs[j - 1], serial[j - 1])
    evs[-1].synchronize()
    assert torch.equal(outs[-1], serial[-1])
    assert binding.get_device_error() == 0
