"""GPU parity of the cache-side kernels (bit-exact against the oracle)."""
import numpy as np
import pytest
import torch

from oracle import cache_ops as ocache
from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem, step_inputs

pytestmark = pytest.mark.gpu


def _bits(t):
    t = t.detach().cpu()
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).numpy()


def _np_bits(a, dtype):
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == torch.bfloat16:
        return (a.view(np.uint32) >> 16).astype(np.uint16).view(np.int16)
    return a.view(np.int32)


def _canon_nan(bits, dtype):
    # every NaN pattern compares as one canonical NaN
    b = bits.copy()
    if dtype == torch.bfloat16:
        nan = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
        b[nan] = 0x7FC0
    else:
        nan = ((b & 0x7F800000) == 0x7F800000) & ((b & 0x7FFFFF) != 0)
        b[nan] = 0x7FC00000
    return b


@pytest.mark.parametrize("name", ["tiny_fp32", "shared_prefix"])
def test_prefill_append_whole_pool_bit_exact(name):
    """Every byte of both caches after the prompts and one decode append,
    compared with the oracle's scatter over a NaN-filled pool."""
    w = wl.WORKLOADS[name]
    cache, lens = gpu_problem(w)
    op = OracleProblem(w, dense=True)
    q, kn, vn = step_inputs(w, 0)
    cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale)
    op.decode_step(0)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    dt = cache.k_cache.dtype
    for dev_c, ora_c in ((cache.k_cache, op.kc), (cache.v_cache, op.vc)):
        got = _canon_nan(_bits(dev_c).reshape(-1), dt)
        exp = _canon_nan(_np_bits(ora_c, dt).reshape(-1), dt)
        assert np.array_equal(got, exp)


def test_walkthrough_slots_written():
    """The 7-token, block-size-4 walkthrough: positions 7 and 8 land in block 1
    offset 3 and block 3 offset 0 (tables [7,1] -> [7,1,3])."""
    # block_size 4 is not a decode-kernel size, but the append and copy kernels take any block size
    nb, bs, hkv, d = 8, 4, 2, 8
    bm = binding.BlockManager(nb, bs, [7, 1, 3, 0, 2, 4, 5, 6])
    kc = torch.full((nb, bs, hkv, d), -7.0, device="cuda")
    vc = torch.full((nb, bs, hkv, d), -7.0, device="cuda")
    k = torch.randn(9, hkv, d, device="cuda")
    v = torch.randn(9, hkv, d, device="cuda")
    slots = list(bm.allocate(0, 7)) + [int(bm.append_slots([0])[0][0]) for _ in range(2)]
    assert slots[7:] == [7, 12]
    binding.reshape_and_cache(k, v, kc, vc, torch.tensor(slots, device="cuda"))
    ko, vo = np.full((nb, bs, hkv, d), -7.0, np.float32), np.full((nb, bs, hkv, d), -7.0, np.float32)
    ocache.reshape_and_cache(k.cpu().numpy(), v.cpu().numpy(), ko, vo, np.asarray(slots))
    assert np.array_equal(kc.cpu().numpy(), ko) and np.array_equal(vc.cpu().numpy(), vo)
    assert torch.equal(kc[1, 3], k[7]) and torch.equal(kc[3, 0], k[8])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_negative_slots_skipped_and_out_of_range_flagged(dtype):
    nb, bs, hkv, d = 6, 16, 4, 64
    kc = torch.zeros((nb, bs, hkv, d), dtype=dtype, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones((4, hkv, d), dtype=dtype, device="cuda")
    slots = torch.tensor([-1, 5, nb * bs, 17], device="cuda")          # pad, ok, out of range, ok
    assert binding.get_device_error() == 0
    binding.reshape_and_cache(k, 2 * k, kc, vc, slots)
    assert binding.get_device_error() == 4
    assert binding.get_device_error() == 0                              # read clears it
    assert kc.sum().item() == 2 * hkv * d and vc.sum().item() == 4 * hkv * d
    assert kc[0, 5].eq(1).all() and kc[1, 1].eq(1).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("hkv,d", [(8, 64), (32, 128), (8, 128)])
def test_copy_blocks_bit_exact(dtype, hkv, d):
    nb, bs = 64, 16
    g = torch.Generator(device="cuda").manual_seed(3)
    kc = torch.randn((nb, bs, hkv, d), generator=g, device="cuda").to(dtype)
    vc = torch.randn((nb, bs, hkv, d), generator=g, device="cuda").to(dtype)
    ko, vo = kc.float().cpu().numpy(), vc.float().cpu().numpy()
    src, dst = [1, 5, 9, 13, 2], [3, 40, 41, 63, 0]
    binding.copy_blocks(kc, vc, torch.tensor(src, device="cuda"), torch.tensor(dst, device="cuda"))
    ocache.copy_blocks(ko, vo, src, dst)
    assert np.array_equal(kc.float().cpu().numpy(), ko) and np.array_equal(vc.float().cpu().numpy(), vo)
    assert binding.get_device_error() == 0


def test_copy_blocks_bad_ids_flagged_and_skipped():
    nb, bs, hkv, d = 8, 16, 2, 64
    kc = torch.zeros((nb, bs, hkv, d), device="cuda")
    vc = torch.zeros_like(kc)
    kc[1] = 1.0
    binding.copy_blocks(kc, vc, torch.tensor([1, -3, 1], device="cuda"), torch.tensor([2, 4, 99], device="cuda"))
    assert binding.get_device_error() == 4
    assert kc[2].eq(1).all() and kc[4].eq(0).all() and kc.sum().item() == 2 * bs * hkv * d


def test_shared_prefix_cow_copies_bit_exact():
    """Parallel-sampling workload: the last shared prefix block is forked for
    all but one sequence, the copies land where the oracle puts them."""
    w = wl.WORKLOADS["shared_prefix"]
    cache, lens = gpu_problem(w)
    op = OracleProblem(w, dense=True)
    last = w.shared_prefix // w.block_size - 1
    pairs = cache.make_writable(list(range(w.num_seqs)), last)
    assert pairs == op.fork_last_shared_block() and len(pairs) == w.num_seqs - 1
    torch.cuda.synchronize()
    dt = cache.k_cache.dtype
    for dev_c, ora_c in ((cache.k_cache, op.kc), (cache.v_cache, op.vc)):
        got = _canon_nan(_bits(dev_c).reshape(-1), dt)
        exp = _canon_nan(_np_bits(ora_c, dt).reshape(-1), dt)
        assert np.array_equal(got, exp)
