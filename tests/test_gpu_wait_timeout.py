"""Bounded waits inside the kernels give up cleanly.

Every mbarrier wait in the decode and tcgen05 multi-query kernels is bounded:
when a copy never lands, the waiting thread gives up, the launch records
PKV_ERR_DEVICE_TIMEOUT in the device error word, drains the copies it did
issue, frees its tensor memory and returns. These tests make one wait run out
without faulting anything: the library's test hook tells the next launch to
never issue one copy (so nothing is left in flight) and to give up after 5 ms.
They check the error word, that the launch returned (the stream synchronises
without a CUDA error), and that the next normal call on the same stream gives
the oracle's result, bit-identical to a call made before the failure (the
tcgen05 kernel's 512 tensor-memory columns were released: a leaked allocation
would stall the next launch instead).
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_322_b200 import binding
from tests.test_gpu_multi_query import _mq_problem, _run

pytestmark = pytest.mark.gpu

LIMIT_NS = 5_000_000          # 5 ms
TIMEOUT = 6                   # PKV_ERR_DEVICE_TIMEOUT


def _decode(dev, part=0):
    out = torch.empty(dev["q"].shape, dtype=torch.float32, device="cuda")
    binding.paged_attention_decode(out, dev["q"], dev["kc"], dev["vc"], dev["tables"], dev["lens"], dev["scale"],
                                   partition_tokens=part)
    return out


@pytest.mark.parametrize("hq,hkv,d", [(8, 8, 128), (32, 4, 128), (4, 4, 64)])
def test_decode_wait_runs_out_then_next_call_is_exact(hq, hkv, d):
    """The first CTA (sequence 0, 200 tokens = 13 ring stages) never gets stage
    2: the consumer waiting for it gives up. MHA (CUDA-core consumers), group 8
    (mma.sync consumers) and head_dim 64."""
    ctxs = [200, 37, 500]
    dev, ref = _mq_problem(31, hq, hkv, d, 16, ctxs, [1, 1, 1])
    good = _decode(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(good.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3

    binding.test_withhold_copy(binding.WITHHOLD_DECODE, 2, LIMIT_NS)
    _decode(dev)
    torch.cuda.synchronize()                     # the launch returned; the context is usable
    assert binding.get_device_error() == TIMEOUT

    again = _decode(dev)                         # the hook was one-shot
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert torch.equal(again, good)


def test_decode_unit_loop_wait_runs_out_then_next_call_is_exact():
    """64-token partitions over contexts up to 900 tokens: 8 or more partitions per
    context, so the partition kernel's unit-loop build runs (about one wave of
    CTAs, each taking several listed units with the ring's phases carried between
    them). The first CTA's first unit never gets ring stage 2: its consumer gives
    up, the CTA drains and leaves its loop, and the next call is exact."""
    ctxs = [600, 900, 500, 130]
    dev, ref = _mq_problem(33, 32, 4, 128, 16, ctxs, [1, 1, 1, 1])
    good = _decode(dev, part=64)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(good.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3

    binding.test_withhold_copy(binding.WITHHOLD_DECODE, 2, LIMIT_NS)
    _decode(dev, part=64)
    torch.cuda.synchronize()
    assert binding.get_device_error() == TIMEOUT

    again = _decode(dev, part=64)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert torch.equal(again, good)


def test_tcgen05_wait_runs_out_then_tensor_memory_is_free():
    """Group 8, 64 query tokens on a 600-token context: the first CTA's query
    tile sees 552 tokens (5 KV tiles of 128); its producer never issues K of
    tile 2, so the MMA thread's wait gives up, then the softmax warps' and the
    producer's. The next call runs on the same stream and must be exact."""
    ctxs, ns = [600, 300], [64, 40]
    dev, ref = _mq_problem(32, 64, 8, 128, 16, ctxs, ns)
    good = _run(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert np.abs(good.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3

    binding.test_withhold_copy(binding.WITHHOLD_MULTI_QUERY_TC, 2, LIMIT_NS)
    _run(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == TIMEOUT

    for _ in range(2):                           # every SM's tensor memory is free again
        again = _run(dev)
        torch.cuda.synchronize()
        assert binding.get_device_error() == 0
        assert torch.equal(again, good)


def test_hook_on_a_stage_the_launch_never_reaches_changes_nothing():
    """Withholding a stage past the first CTA's last one is a no-op (the hook is
    still consumed): no timeout, the exact result."""
    ctxs = [40, 300]
    dev, ref = _mq_problem(33, 8, 8, 128, 16, ctxs, [1, 1])
    good = _decode(dev)
    binding.test_withhold_copy(binding.WITHHOLD_DECODE, 50, LIMIT_NS)
    again = _decode(dev)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    assert torch.equal(again, good)
    assert np.abs(good.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3
