"""Full-size workloads on the GPU, in the launch configuration the benchmark
times: sampled sequences against the oracle, and properties that hold for
every sequence at any size."""
import numpy as np
import pytest
import torch

from paged_kv_cache_322_b200 import binding, workloads as wl
from tests.paged_problem import OracleProblem, gpu_problem, step_inputs, tolerance

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,part", [("llama2_7b", 0), ("llama2_13b", 0), ("gqa_70b", 0), ("shared_prefix", 0),
                                       ("long_splitk", 512),
                                       ("long_splitk", -1), ("llama2_7b", -1), ("gqa_70b", -1)])
def test_full_size_sampled_against_oracle(name, part):
    """part 0: library-chosen partitions; 512: fixed 512-token partitions;
    -1: the persistent schedule."""
    import dataclasses
    w = dataclasses.replace(wl.WORKLOADS[name], partition_tokens=part)
    sample = wl.sample_seqs(w, 6)
    cache, lens = gpu_problem(w, fill_nan=(name == "shared_prefix"))
    op = OracleProblem(w, keep=sample)
    if name == "shared_prefix":
        pairs = cache.make_writable(list(range(w.num_seqs)), w.shared_prefix // w.block_size - 1)
        assert pairs == op.fork_last_shared_block()
    q, kn, vn = step_inputs(w, 0)
    out = cache.decode_step(np.arange(w.num_seqs), q, kn, vn, w.scale, out_dtype=torch.float32,
                            partition_tokens=w.partition_tokens)
    ref = op.decode_step(0, seqs=sample)
    torch.cuda.synchronize()
    assert binding.get_device_error() == 0
    got = out.cpu().numpy()
    err = np.abs(got[sample].astype(np.float64) - ref).max()
    assert err <= tolerance(w), err
    # every sequence: finite, and a convex combination of values bounds each output
    assert np.isfinite(got).all()
    assert np.abs(got).max() <= 6.0
    # bf16 output, same launch: agrees with the fp32 output to bf16 rounding
    out_bf = cache_rerun(cache, q, w)
    assert np.all(np.abs(out_bf - got) <= np.abs(got) * 2 ** -8 + 1e-6)


def cache_rerun(cache, q, w):
    """Attention again over the same (already appended) state, bf16 output."""
    tables, lens = cache.block_tables(np.arange(w.num_seqs))
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    binding.paged_attention_decode(out, q, cache.k_cache, cache.v_cache, torch.from_numpy(tables).cuda(),
                                   torch.from_numpy(lens).cuda(), w.scale, max_context_len=int(lens.max()),
                                   partition_tokens=w.partition_tokens)
    return out.float().cpu().numpy()
